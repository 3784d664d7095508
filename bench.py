"""Benchmark of the CubicQuant weight-only GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl cuda|reference]
                    [--workload down_m1|gate_up_m1|...] [--no-secondary]

Headline workload (default): the Kimi-K3-shaped expert down_proj stored as
CubicQuant W3 G512, N = 7168 x K = 3072, one activation row (M = 1).  One
step is one fused GEMM (unpack -> level generation -> tcgen05 MMA -> output)
over one weight copy; consecutive steps rotate through R distinct copies
whose total size exceeds 4x the L2 cache, so every step streams its packed
weights from HBM.  Metric: packed-weight GB/s = N*K*(B + 64/G)/8 bytes per
step / time per step (x and y excluded, as the metric defines it).

Timing: W untimed warm-up steps, then exactly K steps captured in one CUDA
graph and bracketed by CUDA events on the launching stream, with a barrier
and device synchronisation on both sides; under torchrun each rank runs its
own replica (no collective on the data path) and the slowest rank's time is
used.  Rank 0 prints one JSON line.

--impl reference runs the CPU oracle (FP64, plain C) on a bounded sample of
the same workload instead, as the reference arm.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

METRIC = "Cubic GEMM packed-weight GB/s at M=1 and TFLOP/s at M>=256, % of B200 roofline"

_DOWN = "Kimi-K3 expert down_proj, CubicQuant W3 G512, N=7168 x K=3072"
_GU = "Kimi-K3 expert gate+up, CubicQuant W2 G512, N=6144 x K=7168, SwiGLU"
WORKLOADS = {
    # name: (description, N, K, B, G, M, epilogue)
    "down_m1": (f"{_DOWN}, M=1", 7168, 3072, 3, 512, 1, 0),
    "down_m4": (f"{_DOWN}, M=4", 7168, 3072, 3, 512, 4, 0),
    "down_m16": (f"{_DOWN}, M=16", 7168, 3072, 3, 512, 16, 0),
    "gate_up_m1": (f"{_GU}, M=1", 6144, 7168, 2, 512, 1, 1),
    "gate_up_m16": (f"{_GU}, M=16", 6144, 7168, 2, 512, 16, 1),
    "gate_up_m64": (f"{_GU}, M=64", 6144, 7168, 2, 512, 64, 1),
    # the M >= 256 clause of the metric on single-matrix shapes (an extension of
    # the configurations: same matrices, larger token counts)
    "down_m256": (f"{_DOWN}, M=256", 7168, 3072, 3, 512, 256, 0),
    "gate_up_m1024": (f"{_GU}, M=1024", 6144, 7168, 2, 512, 1024, 1),
    "gate_up_m4096": (f"{_GU}, M=4096", 6144, 7168, 2, 512, 4096, 1),
    "down_m4096": (f"{_DOWN}, M=4096", 7168, 3072, 3, 512, 4096, 0),
    # the Dynamic A8 path (INT8 activations) beside A16, where the article
    # reports the crossover ("实验结果 2. H200 内核交叉点")
    "a8_gate_up_m64": (f"Dynamic A8: {_GU}, M=64", 6144, 7168, 2, 512, 64, 1),
    "a8_down_m256": (f"Dynamic A8: {_DOWN}, M=256", 7168, 3072, 3, 512, 256, 0),
    "a8_gate_up_m4096": (f"Dynamic A8: {_GU}, M=4096", 6144, 7168, 2, 512, 4096, 1),
}
# the GEMM lines printed under "secondary", in order
SECONDARY = ["down_m4", "down_m16", "gate_up_m1", "gate_up_m16", "gate_up_m64", "down_m256",
             "gate_up_m1024", "gate_up_m4096", "down_m4096", "a8_gate_up_m64", "a8_down_m256",
             "a8_gate_up_m4096"]
NOMINAL_HBM_GBS = 8000.0          # the ~8 TB/s HBM3e figure
NOMINAL_BF16_TFLOPS = 2250.0      # dense BF16 datasheet figure


# DRAM bytes (read + write) per launch of the dominant kernel, from one ncu capture.
# Keyed by the SHA-256 of the kernel's sources at capture time: once they change,
# the figure no longer describes the kernel and `traffic` is reported as null.
KERNEL_SOURCES = ("cq_gemv.cuh", "cq_gemv_launch.cuh", "cq_device.cuh")
TRAFFIC = {
    "down_m1": {"kernel": "gemv_kernel<3,1>", "bytes": 8652544,
                "sources_sha256": "4bc21cfec1c73681d65a8f2cb03f13c3d0e85f9274f572aa73c0908e38002910"},
}


def kernel_sources_sha256():
    import hashlib
    h = hashlib.sha256()
    for name in KERNEL_SOURCES:
        with open(os.path.join(ROOT, "bit_non_uniform_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def measured_traffic(name):
    rec = TRAFFIC.get(name)
    if rec is None or rec["sources_sha256"] != kernel_sources_sha256():
        return None
    return rec["bytes"]


def main_roofline(r, ach_gbs, hbm, tf_burst, traffic, name, peak_src):
    """The roofline of the main line's kernel: HBM for the decode-sized
    workloads, the BF16 tensor peak (burst: one kernel timed alone) for
    M >= 256."""
    if r["M"] >= 256:
        return {"bound": "tensor", "achieved": round(r["tflops"], 1), "peak": tf_burst,
                "unit": "TFLOP/s", "frac": round(r["tflops"] / tf_burst, 4), "traffic": traffic,
                "kernel": dominant_kernel(name), "peak_source": peak_src}
    return {"bound": "hbm", "achieved": round(ach_gbs, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(ach_gbs / hbm, 4), "traffic": traffic,
            "kernel": dominant_kernel(name), "peak_source": peak_src}


def dominant_kernel(name):
    """The kernel one cq_gemm launch of the workload runs (the only one it runs)."""
    _, N, K, B, G, M, epi = WORKLOADS[name]
    if name.startswith("a8_"):
        nt = 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128
        return f"quant_rows_kernel + engine_a8_kernel<{nt},{64 if B == 3 else 16}>"
    if M <= 2:
        return f"gemv_kernel<{B},{M}>"
    if M <= 8 and K % 512 == 0 and 2 <= B <= 4:
        return f"narrow_kernel<{B},8>"
    if M <= 128:
        nt = 16 if M <= 16 else 32 if M <= 32 else 64 if M <= 64 else 128
    else:
        pad128 = -(-M // 128) * 128
        if B == 3:
            nt = 176 if -(-M // 176) * 176 * 100 <= pad128 * 105 else 128
        else:
            nt = 192 if -(-M // 192) * 192 * 100 <= pad128 * 115 else 128
    return f"engine_kernel<{nt},{64 if B == 3 else 16}>"


def packed_bytes(N, K, B, G):
    return N * K * B // 8 + N * (K // G) * 8


def load_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(
            d.get("bf16_tflops_sustained", d["bf16_tflops"])), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


# --------------------------------------------------------------------------
# clock sampling (NVML) during the timed region
# --------------------------------------------------------------------------

class ClockSampler:
    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int):
        self.samples, self.reasons = [], 0
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nvml = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception:
            self.max_mhz = None
        self._stop = threading.Event()

    def _poll(self):
        n = self.nvml
        while not self._stop.is_set():
            try:
                self.samples.append(n.nvmlDeviceGetClockInfo(self.h, n.NVML_CLOCK_SM))
                self.reasons |= n.nvmlDeviceGetCurrentClocksEventReasons(self.h)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self.ok:
            self._sample_once()
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
        return self

    def _sample_once(self):
        try:
            self.samples.append(self.nvml.nvmlDeviceGetClockInfo(self.h, self.nvml.NVML_CLOCK_SM))
            self.reasons |= self.nvml.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()
            self._sample_once()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [k for k, v in self.REASONS.items() if self.reasons & v]}


# --------------------------------------------------------------------------
# distributed plumbing (replicas only; no data-path collective)
# --------------------------------------------------------------------------

def dist_setup(args):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v: float, world: int) -> float:
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, ms_per_rank: float, world: int) -> float:
    """Whole-job throughput of replicas: every rank processes the same units,
    the job takes as long as the slowest rank (units per ms, all ranks)."""
    slowest = max_over_ranks(ms_per_rank, world)
    return units_per_rank * world / slowest


# --------------------------------------------------------------------------
# GPU arm
# --------------------------------------------------------------------------

def build_weights(cq, name, device):
    import synthetic
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    codes, s, ab = synthetic.matrix(("bench", name), N, K, B, G, device=device)
    packed = cq.cq_pack(codes, B)
    del codes
    return packed, s.contiguous(), ab.contiguous()


def rotation_copies(nbytes, l2_bytes):
    return max(2, int(np.ceil(4.5 * l2_bytes / nbytes)))


# Cycles of the spin kernel queued ahead of the first timing event: it keeps the
# GPU busy while the host enqueues the graph replay, so the timed region holds the
# launches only, whatever the host-side latency of the replay call (about 0.5 ms
# at the 1.9 GHz clock; much longer than any enqueue).
SPIN_CYCLES = 1_000_000


def timed_replay(g, stream):
    """Milliseconds of one replay of graph g, CUDA events on `stream`, with a
    spin kernel queued ahead of the first event."""
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        torch.cuda._sleep(SPIN_CYCLES)
        ev0.record(stream)
        g.replay()
        ev1.record(stream)
    ev1.synchronize()
    return ev0.elapsed_time(ev1)


def time_gemm(cq, name, steps, warmup, world, device, sample_clocks=False, repeats=0):
    """Device-timed K steps of one workload (CUDA graph of K launches)."""
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    import synthetic
    packed, s, ab = build_weights(cq, name, device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    wbytes = packed_bytes(N, K, B, G)
    R = rotation_copies(wbytes, l2) if M <= 64 else 1
    copies = [(packed.clone(), s.clone(), ab.clone()) for _ in range(R)]
    x = synthetic.activations(11, M, K).to(device)
    ncol = N // 2 if epi else N
    y = torch.empty((M, ncol), dtype=torch.float32, device=device)
    a8 = name.startswith("a8_")
    if a8:
        n = cq.gemm_a8_workspace_size(M, N, K, B, G, epi)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=device)
    else:
        ws = cq.gemm_workspace(M, N, K, B, G, epi, device)
    stream = torch.cuda.Stream(device)

    def step(i, st):
        p, sc, a = copies[i % R]
        if a8:
            cq.cq_gemm_a8(x, p, sc, a, N, K, B, G, epilogue=epi, workspace=ws, out=y, stream=st)
        else:
            cq.cq_gemm(x, p, sc, a, N, K, B, G, epilogue=epi, workspace=ws, out=y, stream=st)

    with torch.cuda.stream(stream):
        for i in range(max(warmup, 3)):
            step(i, stream)
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for i in range(steps):
            step(i, stream)
    # one untimed replay (graph upload) before timing
    g.replay()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    sampler = ClockSampler(device.index if device.index is not None else 0)
    with sampler if sample_clocks else _null():
        ms = timed_replay(g, stream)
    torch.cuda.synchronize()
    barrier(world)
    ms = max_over_ranks(ms, world)
    reps = []
    if repeats:
        for _ in range(repeats):
            reps.append(timed_replay(g, stream) / steps)
        torch.cuda.synchronize()
    st, site = cq.device_error()
    if st != 0:
        raise RuntimeError(f"device wait timed out (site {site})")
    del g
    flops = 2.0 * M * N * K
    res = dict(name=name, desc=desc, M=M, N=N, K=K, B=B, G=G, epilogue=epi, R=R,
               rot_mb=R * wbytes / 1e6, ms_total=ms, ms_per_step=ms / steps,
               wbytes=wbytes, gbs=wbytes * steps / (ms * 1e-3) / 1e9,
               tflops=flops * steps / (ms * 1e-3) / 1e12,
               alg_bytes=wbytes + M * K * 2 + M * ncol * 4,
               clocks=sampler.summary() if sample_clocks else None)
    if reps:
        res["rep_ms_per_step"] = sorted(reps)
    return res


def gemm_entry(r, hbm, tf_burst, world):
    """One secondary line: HBM roofline up to M = 64, BF16 tensor above."""
    ent = {"workload": r["desc"], "ms_per_step": round(r["ms_per_step"], 6),
           "packed_gbs": round(r["gbs"] * world, 1), "tflops": round(r["tflops"] * world, 2),
           "kernel": dominant_kernel(r["name"]),
           "l2": f"{r['R']} rotating weight copies ({r['rot_mb']:.0f} MB)"}
    if "rep_ms_per_step" in r:
        ent["best_ms_per_step"] = round(min(r["rep_ms_per_step"]), 6)
        ent["median_ms_per_step"] = round(statistics.median(r["rep_ms_per_step"]), 6)
    if r["M"] <= 64:
        ach = r["alg_bytes"] / (r["ms_per_step"] * 1e-3) / 1e9
        ent["roofline"] = {"bound": "hbm", "achieved": round(ach, 1), "peak": hbm,
                           "unit": "GB/s", "frac": round(ach / hbm, 4),
                           "frac_nominal": round(ach / NOMINAL_HBM_GBS, 4)}
    elif r["name"].startswith("a8_"):
        # INT8 tensor peak: the measured BF16 peak times the nominal 2x ratio
        pk = 2.0 * tf_burst
        ent["roofline"] = {"bound": "tensor", "achieved": round(r["tflops"], 1),
                           "peak": round(pk, 1), "unit": "TOP/s",
                           "frac": round(r["tflops"] / pk, 4),
                           "frac_nominal": round(r["tflops"] / (2 * NOMINAL_BF16_TFLOPS), 4),
                           "peak_kind": "int8 = 2 x the measured bf16 peak"}
    else:
        ent["roofline"] = {"bound": "tensor", "achieved": round(r["tflops"], 1),
                           "peak": tf_burst, "unit": "TFLOP/s",
                           "frac": round(r["tflops"] / tf_burst, 4),
                           "frac_nominal": round(r["tflops"] / NOMINAL_BF16_TFLOPS, 4)}
    return ent


def time_cold(cq, name, device):
    """One launch on a cold cache: L2 flushed by writing a buffer larger than
    it, the GPU idle, an ordinary (non-graph) call.  Reports the CUDA-event
    time on the stream (launch latency on the device included) and the host
    wall time of the call plus synchronisation."""
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    import synthetic
    packed, s, ab = build_weights(cq, name, device)
    x = synthetic.activations(13, M, K).to(device)
    y = torch.empty((M, N // 2 if epi else N), dtype=torch.float32, device=device)
    ws = cq.gemm_workspace(M, N, K, B, G, epi, device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    flush = torch.empty(int(2 * l2), dtype=torch.uint8, device=device)
    stream = torch.cuda.Stream(device)
    with torch.cuda.stream(stream):
        cq.cq_gemm(x, packed, s, ab, N, K, B, G, epilogue=epi, workspace=ws, out=y,
                   stream=stream)        # module and first-call setup, not timed
        flush.fill_(1)
    stream.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.perf_counter()
    ev0.record(stream)
    cq.cq_gemm(x, packed, s, ab, N, K, B, G, epilogue=epi, workspace=ws, out=y, stream=stream)
    ev1.record(stream)
    ev1.synchronize()
    wall = time.perf_counter() - t0
    return {"device_us": round(ev0.elapsed_time(ev1) * 1e3, 2), "host_wall_us": round(wall * 1e6, 1),
            "l2_flushed_bytes": int(flush.numel())}


MOE_WORKLOADS = {
    # name: (description, T, routing, widths, experts)
    "moe_decode": ("Kimi-K3 MoE layer, 896 experts W2/W3/W4 (P=.6/.3/.1) G512, 64 tokens, "
                   "uniform top-16", 64, "uniform", "mixed", 896),
    "moe_prefill": ("Kimi-K3 MoE layer, 896 experts W4 G512, 8192 tokens, Zipf(1.1) top-16",
                    8192, "zipf", "w4", 896),
    # the decode layer's kernels on 64 of its experts (1.3 GB of weights: a size an ncu
    # capture with every counter can replay); not a bench line
    "moe_decode_64e": ("Kimi-K3 MoE layer shapes, 64 experts W2/W3/W4 (P=.6/.3/.1) G512, "
                       "16 tokens, uniform top-16", 16, "uniform", "mixed", 64),
}


def time_moe(cq, name, steps, device):
    """Device-timed steps of one MoE layer (routing, gather, gate/up, down,
    combine), captured in a CUDA graph; inputs and weights resident."""
    import synthetic
    desc, T, routing, widths, E = MOE_WORKLOADS[name]
    H, I, k, G = 7168, 3072, 16, 512
    Bs = synthetic.expert_bits(4, E) if widths == "mixed" else torch.full((E,), 4)
    experts = []
    for e in range(E):
        B = int(Bs[e])
        gu = synthetic.matrix(("bench", name, "gu", e), 2 * I, H, B, G, device=device)
        dn = synthetic.matrix(("bench", name, "dn", e), H, I, B, G, device=device)
        experts.append(dict(B_gu=B, packed_gu=cq.cq_pack(gu[0], B), scales_gu=gu[1],
                            ab_gu=gu[2], B_dn=B, packed_dn=cq.cq_pack(dn[0], B),
                            scales_dn=dn[1], ab_dn=dn[2]))
        del gu, dn
    layer = cq.moe_prepare_layer(experts, H, I, G, device)
    x = synthetic.activations(7, T, H).to(device)
    if routing == "uniform":
        ids, w = synthetic.routing_uniform(4, T, E, k)
    else:
        ids, w = synthetic.routing_zipf(5, T, E, k)
    ids_d, w_d = ids.to(device), w.to(device)
    ws = cq.moe_workspace(T, k, E, H, I, G, device)
    out = torch.empty((T, H), dtype=torch.float32, device=device)
    stream = torch.cuda.Stream(device)
    lib = cq.lib()

    def step():
        st = lib.cq_moe_grouped_gemm(
            cq._ptr(x), T, cq._ptr(ids_d), cq._ptr(w_d), k, E, cq._ptr(layer), H, I, G, 0, 0,
            None, cq._ptr(out), cq._ptr(ws), ws.numel(), cq._stream(stream))
        if st != 0:
            raise RuntimeError(f"cq_moe_grouped_gemm status {st}")

    with torch.cuda.stream(stream):
        for _ in range(3):
            step()
    stream.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for _ in range(steps):
            step()
    g.replay()
    torch.cuda.synchronize()
    ms = timed_replay(g, stream) / steps
    st, site = cq.device_error()
    if st != 0:
        raise RuntimeError(f"device wait timed out (site {site})")
    del g
    active = torch.unique(ids).tolist()
    wbytes = sum(packed_bytes(2 * I, H, int(Bs[e]), G) + packed_bytes(H, I, int(Bs[e]), G)
                 for e in active)
    flops = 2.0 * T * k * (2 * I * H + H * I)
    mean_bits = sum(int(Bs[e]) for e in active) / len(active)
    return dict(name=name, desc=desc, ms=ms, tokens_per_s=T / (ms * 1e-3),
                gbs=wbytes / (ms * 1e-3) / 1e9, tflops=flops / (ms * 1e-3) / 1e12,
                active=len(active), wbytes=wbytes, mean_payload_bits=mean_bits)


class _null:
    def __enter__(self):
        return self

    def __exit__(self, *a):
        return False


def time_e2e(cq, name, steps, device):
    """End to end through the C ABI with host buffers: per step one
    cq_gemm_host call, which queues the copy of the pinned-host x into a
    device staging buffer, the GEMM and the copy of y into pinned host memory
    (ordinary calls, not a graph; the ctypes arguments are marshalled once)."""
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    import ctypes
    import synthetic
    packed, s, ab = build_weights(cq, name, device)
    l2 = torch.cuda.get_device_properties(device).L2_cache_size
    wbytes = packed_bytes(N, K, B, G)
    R = rotation_copies(wbytes, l2) if M <= 64 else 1
    copies = [(packed.clone(), s.clone(), ab.clone()) for _ in range(R)]
    xh = synthetic.activations(12, M, K).pin_memory()
    ncol = N // 2 if epi else N
    yh = torch.empty((M, ncol), dtype=torch.float32).pin_memory()
    xd = torch.empty((M, K), dtype=torch.bfloat16, device=device)
    yd = torch.empty((M, ncol), dtype=torch.float32, device=device)
    ws = cq.gemm_workspace(M, N, K, B, G, epi, device)
    stream = torch.cuda.Stream(device)
    n = max(10, min(steps, 2000))
    f = cq.lib().cq_gemm_host
    P = ctypes.c_void_p
    args = [(P(xh.data_ptr()), M, P(p.data_ptr()), P(sc.data_ptr()), P(a.data_ptr()), N, K, B, G,
             cq.MIDRISE, epi, cq.F32, P(yh.data_ptr()), P(xd.data_ptr()), P(yd.data_ptr()),
             P(ws.data_ptr()), ws.numel(), P(stream.cuda_stream)) for p, sc, a in copies]

    def one(i):
        st = f(*args[i % R])
        if st != 0:
            raise RuntimeError(f"cq_gemm_host returned {st}")

    for i in range(5):
        one(i)
    stream.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    ev0.record(stream)
    t0 = time.perf_counter()
    for i in range(n):
        one(i)
    ev1.record(stream)
    ev1.synchronize()
    wall = time.perf_counter() - t0
    ms = ev0.elapsed_time(ev1)
    return {"value": round(wbytes * n / (ms * 1e-3) / 1e9, 3), "unit": "GB/s",
            "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * ncol * 4,
            "steps": n, "ms_per_step": ms / n, "host_wall_us_per_step": round(wall / n * 1e6, 2),
            "call": "cq_gemm_host (C ABI, pinned host x and y)"}


# --------------------------------------------------------------------------
# CPU oracle (reference arm and cpu_baseline)
# --------------------------------------------------------------------------

def oracle_sample(name, rows):
    import oracle
    import synthetic
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    codes, s, ab = synthetic.matrix(("bench", name), N, K, B, G, nrows=rows)
    packed = oracle.pack(codes.numpy(), B)
    x = synthetic.activations(11, M, K).view(torch.int16).numpy().view(np.uint16)
    return (oracle, packed, s.numpy(), ab.view(torch.int16).numpy().view(np.uint16), x,
            rows, K, B, G)


def time_oracle(name, rows, min_seconds=0.0, reps=1, nthreads=0):
    oracle, packed, s, ab, x, rows, K, B, G = oracle_sample(name, rows)
    wbytes = packed_bytes(rows, K, B, G)
    n = 0
    t0 = time.perf_counter()
    while True:
        oracle.gemm(x, packed, s, ab, rows, K, B, G, nthreads=nthreads)
        n += 1
        el = time.perf_counter() - t0
        if n >= reps and el >= min_seconds:
            break
    return wbytes * n / el / 1e9, el, n, oracle.num_threads()


def cpu_baseline(name):
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    gbs, el, n, cores = time_oracle(name, N, min_seconds=10.0)
    return {"value": round(gbs, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"the full {N}x{K} W{B} G{G} matrix at M={M}, {n} pass(es), "
                      f"{el:.1f} s, FP64 plain C over {cores} threads"}


def _oracle_expert(tag, e, B, H, I, G, device):
    """One expert's matrices from the seeded generator (drawn on the GPU, the
    same values as on the CPU), packed by the oracle on the host."""
    import oracle
    import synthetic
    u16 = lambda t: t.cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    gu = [t.cpu() for t in synthetic.matrix((tag, "gu", e), 2 * I, H, B, G, device=device)]
    dn = [t.cpu() for t in synthetic.matrix((tag, "dn", e), H, I, B, G, device=device)]
    return dict(B_gu=B, packed_gu=oracle.pack(gu[0].numpy(), B), scales_gu=gu[1].numpy(),
                ab_gu=u16(gu[2]), B_dn=B, packed_dn=oracle.pack(dn[0].numpy(), B),
                scales_dn=dn[1].numpy(), ab_dn=u16(dn[2]))


def cpu_baselines(device):
    """The oracle (FP64, plain C, all host threads unless stated) on bounded
    samples of the other configurations, with what each sample was.  Timed:
    the oracle's products only (input generation and packing excluded)."""
    import oracle
    import synthetic
    out = []
    cores = oracle.num_threads()
    # config 1: the fitted W4 G128 256 x 1024 matrix at M = 1, in full
    d = np.load(os.path.join(ROOT, "tests", "golden", "config1_w4g128.npz"))
    x1 = synthetic.activations(1, 1, 1024).view(torch.int16).numpy().view(np.uint16)
    n, t0 = 0, time.perf_counter()
    while n < 3 or time.perf_counter() - t0 < 2.0:
        oracle.gemm(x1, d["packed"], d["scales"], d["ab"], 256, 1024, 4, 128)
        n += 1
    el = time.perf_counter() - t0
    out.append({"config": "W4 G128 256x1024 fitted (config 1), M=1", "value":
                round(packed_bytes(256, 1024, 4, 128) * n / el / 1e9, 4), "unit": "GB/s",
                "cores": cores, "sample": f"the full matrix, {n} passes, {el:.1f} s"})
    # config 3: gate+up W2 at M = 1, 1024 of 6144 rows
    gbs, el, n, _ = time_oracle("gate_up_m1", 1024, min_seconds=2.0)
    out.append({"config": WORKLOADS["gate_up_m1"][0], "value": round(gbs, 4), "unit": "GB/s",
                "cores": cores, "sample": f"1024 of 6144 rows, {n} passes, {el:.1f} s"})
    # config 2 on one core
    gbs, el, n, _ = time_oracle("down_m1", 512, min_seconds=2.0, nthreads=1)
    out.append({"config": WORKLOADS["down_m1"][0], "value": round(gbs, 4), "unit": "GB/s",
                "cores": 1, "sample": f"512 of 7168 rows on one thread, {n} passes, {el:.1f} s"})
    # configs 4 and 5: whole routed-expert chains of sampled experts, scaled by
    # the layer's active experts (the per-expert cost is the decode of its two
    # matrices plus its routes' products)
    H, I, E, k, G = 7168, 3072, 896, 16, 512
    for cfg, T, routing, widths in [("config 4", 64, "uniform", "mixed"),
                                    ("config 5", 8192, "zipf", "w4")]:
        Bs = synthetic.expert_bits(4, E) if widths == "mixed" else torch.full((E,), 4)
        if routing == "uniform":
            ids, _ = synthetic.routing_uniform(4, T, E, k)
        else:
            ids, _ = synthetic.routing_zipf(5, T, E, k)
        ids_np = ids.numpy()
        x = synthetic.activations(7, T, H).view(torch.int16).numpy().view(np.uint16)
        counts = np.bincount(ids_np.ravel(), minlength=E)
        active = np.nonzero(counts)[0]
        sample = [int(active[0]), int(active[len(active) // 2])]
        spent, routes_done, expert_routes = 0.0, 0, 0
        for e in sample:
            ex = _oracle_expert(("cpu", cfg), e, int(Bs[e]), H, I, G, device)
            rs = [int(r) for r in np.nonzero(ids_np.ravel() == e)[0]]
            t0 = time.perf_counter()
            oracle.moe_routes(x, ids_np, {e: ex}, H, I, G, routes=rs)
            spent += time.perf_counter() - t0
            routes_done += len(rs)
        per_expert = spent / len(sample)
        layer_s = per_expert * len(active)
        out.append({"config": f"{cfg}: {T} tokens, top-16 over 896 experts ({widths})",
                    "value": round(T / layer_s, 3), "unit": "tokens/s", "cores": cores,
                    "sample": f"{len(sample)} experts ({routes_done} routes) timed in full, "
                              f"{spent:.1f} s; layer time extrapolated to the "
                              f"{len(active)} active experts ({layer_s:.0f} s)",
                    "extrapolated": True})
    return out


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    name = args.workload
    desc, N, K, B, G, M, epi = WORKLOADS[name]
    rows = min(N, 1024)
    oracle, packed, s, ab, x, rows, K, B, G = oracle_sample(name, rows)
    wbytes = packed_bytes(rows, K, B, G)
    for _ in range(max(args.warmup, 0)):
        oracle.gemm(x, packed, s, ab, rows, K, B, G)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        oracle.gemm(x, packed, s, ab, rows, K, B, G)
    el = time.perf_counter() - t0
    val = wbytes * args.steps / el / 1e9
    cores = oracle.num_threads()
    line = {
        "impl": "reference", "metric": METRIC, "value": round(val, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": desc, "M": M, "N": N, "K": K, "B": B, "G": G},
        "cpu_baseline": {"value": round(val, 4), "unit": "GB/s", "cores": cores,
                         "kind": "oracle",
                         "sample": f"{rows} of {N} weight rows per step at M={M}"},
        "e2e": {"value": round(val, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# --------------------------------------------------------------------------

def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="cuda", choices=["cuda", "reference"])
    ap.add_argument("--workload", default="down_m1", choices=sorted(WORKLOADS))
    ap.add_argument("--no-secondary", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-moe", action="store_true")
    ap.add_argument("--moe-only", choices=sorted(MOE_WORKLOADS),
                    help="time one MoE layer and print its line only (for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        return run_reference(args, world, rank)

    import bit_non_uniform_b200 as cq
    world, rank, local = dist_setup(args)
    device = torch.device("cuda", torch.cuda.current_device())
    hbm, tf_burst, tf_sust, peak_src = load_peaks()
    if args.moe_only:
        r = time_moe(cq, args.moe_only, max(args.steps, 1), device)
        if rank == 0:
            print(json.dumps({"workload": r["desc"], "ms_per_step": round(r["ms"], 4),
                              "active_weight_bytes": r["wbytes"],
                              "packed_gbs": round(r["gbs"], 1), "tflops": round(r["tflops"], 2),
                              "frac_hbm": round(r["gbs"] / hbm, 4)}))
        return 0

    main_res = time_gemm(cq, args.workload, args.steps, args.warmup, world, device,
                         sample_clocks=True, repeats=20)
    secondary = []
    if not args.no_secondary:
        for name in SECONDARY:
            if name == args.workload:
                continue
            steps = 400 if WORKLOADS[name][5] <= 64 else 20
            r = time_gemm(cq, name, steps, 3, world, device, repeats=20)
            secondary.append(gemm_entry(r, hbm, tf_burst, world))
            torch.cuda.empty_cache()

    if not args.no_secondary and not args.no_moe:
        for name in ["moe_decode", "moe_prefill"]:
            r = time_moe(cq, name, 20 if name == "moe_decode" else 5, device)
            ent = {"workload": r["desc"], "ms_per_step": round(r["ms"], 4),
                   "tokens_per_s": round(r["tokens_per_s"] * world, 1),
                   "packed_gbs": round(r["gbs"] * world, 1),
                   "tflops": round(r["tflops"] * world, 2),
                   "active_experts": r["active"],
                   "active_weight_bytes": r["wbytes"],
                   "mean_payload_bits_active": round(r["mean_payload_bits"], 4)}
            if name == "moe_decode":
                ent["roofline"] = {"bound": "hbm", "achieved": round(r["gbs"], 1), "peak": hbm,
                                   "unit": "GB/s", "frac": round(r["gbs"] / hbm, 4),
                                   "frac_nominal": round(r["gbs"] / NOMINAL_HBM_GBS, 4)}
            else:
                ent["roofline"] = {"bound": "tensor", "achieved": round(r["tflops"], 1),
                                   "peak": tf_sust, "unit": "TFLOP/s",
                                   "frac": round(r["tflops"] / tf_sust, 4),
                                   "frac_nominal": round(r["tflops"] / NOMINAL_BF16_TFLOPS, 4),
                                   "peak_kind": "sustained"}
            secondary.append(ent)
            torch.cuda.empty_cache()

    cold = time_cold(cq, args.workload, device)
    e2e = time_e2e(cq, args.workload, args.steps, device)
    e2e["value"] = round(e2e["value"] * world, 3)

    if rank != 0:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return 0

    r = main_res
    value = r["gbs"] * world          # every rank streams its own replica
    ach = r["alg_bytes"] / (r["ms_per_step"] * 1e-3) / 1e9
    traffic = measured_traffic(args.workload)
    line = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(r["ms_per_step"], 6),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": r["desc"], "M": r["M"], "N": r["N"], "K": r["K"],
                   "B": r["B"], "G": r["G"], "bytes_per_step": r["wbytes"],
                   "l2": f"inputs larger than L2: {r['R']} rotating weight copies, "
                         f"{r['rot_mb']:.0f} MB",
                   "parallelism": f"replicas x{world}" if world > 1 else "single GPU"},
        "roofline": main_roofline(r, ach, hbm, tf_burst, traffic, args.workload, peak_src),
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": r["clocks"],
        "timing": {"method": "one replay of a CUDA graph of the K steps, CUDA events on the "
                             "launching stream, a spin kernel queued ahead of the first event",
                   "repeats": len(r.get("rep_ms_per_step", [])),
                   "best_ms_per_step": round(min(r["rep_ms_per_step"]), 6),
                   "median_ms_per_step": round(statistics.median(r["rep_ms_per_step"]), 6),
                   "cold_launch": cold},
        "frac_nominal_hbm": round(ach / NOMINAL_HBM_GBS, 4),
        "secondary": secondary,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(args.workload)
        line["cpu_baselines"] = cpu_baselines(device)
    print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
