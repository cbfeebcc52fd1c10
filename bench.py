#!/usr/bin/env python
"""W4A16 GEMM throughput on B200: HBM GB/s at M=1 and TFLOPS at M=256, against the roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Workload of the headline line: the decode linears of an 80-layer Llama-3-70B-shaped model for
one token, M = 1: per layer (K, N) = (8192, 10240) qkv, (8192, 8192) o, (8192, 57344) gate+up,
(28672, 8192) down; g128 asymmetric INT4; bf16 activations ~ N(0, 1); weights ~ N(0, 0.02).
Four weight matrices are drawn and quantized, and each is copied into 80 distinct device
buffers: one step streams 35.6 GB of packed weights, so L2 (126 MB) cannot serve repeats.
A step is the 320 GEMMs of one token, replayed from a CUDA graph.

Printed (rank 0, one JSON line): value = algorithmic bytes of all ranks' steps / max-over-ranks
device time (GB/s); e2e = the same through the Python API with the step's activations copied
from pinned host memory and its outputs read back; roofline of the dominant kernel (its in-step
time); the FP64 oracle's throughput on the host cores (cpu_baseline); clocks sampled during the
timed region. Extra keys: the 32-layer Llama-3-8B stack, the (8192, 28672) sweep layer at
M = 256 (TFLOPS), the naive dequantize-then-GEMM path, the calibrated encoders, the crossover
sweep against the W8A8 FP8 path, the format variants and the oracle on every configuration.

N > 1 (torchrun): weak scaling, every rank runs its own replica of the workload; no collective
on the data path (NCCL carries only the barrier and the max of the timings).
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

LLAMA8B_LINEARS = (("qkv", 4096, 6144), ("o", 4096, 4096), ("gate_up", 4096, 28672),
                   ("down", 14336, 4096))
LAYERS = 32
LLAMA70B_LINEARS = (("qkv", 8192, 10240), ("o", 8192, 8192), ("gate_up", 8192, 57344),
                    ("down", 28672, 8192))
LAYERS_70B = 80
GROUP = 128
SYM = 0
SWEEP_K, SWEEP_N, SWEEP_M = 8192, 28672, 256
METRIC = "W4A16 GEMM HBM GB/s at M=1 and TFLOPS at M=256, as % of B200 roofline"
SWEEP_MS = (1, 2, 4, 8, 16, 32, 64, 128, 256, 512, 2048)
# ncu DRAM traffic of the decode kernel, written by hand from a capture into this file, with the
# hash of the kernel sources it was taken on (the bench reports it only while they match)
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "gemv_stream_traffic.txt")   # JSON
DECODE_SOURCES = ("gemv_stream.cu", "sm100_ptx.cuh", "tiled_layout.cuh", "common.cuh")


# ----------------------------------------------------------------------------- work model
def algorithmic_bytes(M, K, N, group=GROUP, sym=SYM, act_bytes=2, out_bytes=2):
    """Bytes a W4A16 GEMM must move at least once: codes 0.5 B/weight, an fp16 scale per
    group, an INT4 zero per group (asymmetric), the activations and the output."""
    codes = K * N // 2
    scales = 2 * N * (K // group)
    zeros = 0 if sym else N * (K // group) // 2
    return codes + scales + zeros + act_bytes * M * K + out_bytes * M * N


def gemm_flops(M, K, N):
    return 2 * M * N * K


def step_time_model(params, bits_per_weight, bytes_per_s, flops_per_s, batch):
    """Roofline time of one decode step: max(weight bytes / bandwidth, 2 * params * batch / flops)
    ("INT8 vs INT4 Quantization, in depth", section "Worked example: where the lines cross")."""
    t_mem = params * bits_per_weight / 8 / bytes_per_s
    t_math = 2 * params * batch / flops_per_s
    return max(t_mem, t_math), t_mem, t_math


def crossover_batch(params, bits_per_weight, bytes_per_s, flops_per_s):
    """Batch at which the compute time reaches the memory floor."""
    return (params * bits_per_weight / 8 / bytes_per_s) / (2 * params / flops_per_s)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        p = json.load(open(path))
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]),
                "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


# ----------------------------------------------------------------------------- ranks
def dist_env():
    return int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")), \
        int(os.environ.get("LOCAL_RANK", "0"))


def replica_seed(base, rank):
    """Each rank draws its own replica of the workload (weak scaling)."""
    return base + 7919 * rank


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (identity for one rank)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist

    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": smax, "reasons": ["unsampled"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ----------------------------------------------------------------------------- workload
class DecodeStack:
    """Quantized decode linears (Llama-3-8B-shaped by default), `layers` copies of each, plus
    per-GEMM activations (fp16 or bf16) and outputs."""

    def __init__(self, torch, native, synthetic, seed, layers=LAYERS, M=1, linears=LLAMA8B_LINEARS,
                 bf16=False):
        self.torch, self.native = torch, native
        dev = torch.device("cuda")
        self.M = M
        self.layers = []
        uniq = []
        tdt = torch.bfloat16 if bf16 else torch.float16
        for i, (name, K, N) in enumerate(linears):
            Wb = synthetic.weights_normal(K, N, seed + i)
            W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).to(dev)
            codes, scales, zeros = native.w4a16_quantize(W, GROUP, SYM)
            uniq.append((name, K, N, codes, scales, zeros))
            del W
        self.tiled = tiled_supported(torch, native, uniq[0][1:6])
        for _ in range(layers):
            lay = []
            for (name, K, N, codes, scales, zeros) in uniq:
                w = {"name": name, "K": K, "N": N, "weight_bytes": codes.numel() * 4 +
                     scales.numel() * 2 + (0 if zeros is None else zeros.numel() * 4)}
                if self.tiled:
                    w["tiled"] = native.w4a16_repack(codes, scales, zeros, K, N, GROUP, SYM)
                else:
                    w["codes"], w["scales"] = codes.clone(), scales.clone()
                    w["zeros"] = None if zeros is None else zeros.clone()
                lay.append(w)
            self.layers.append(lay)
        del uniq
        # activations: one flat device buffer (and a pinned host twin for the e2e leg)
        self.a_elems = sum(M * K for (_, K, _) in linears) * layers
        self.c_elems = sum(M * N for (_, _, N) in linears) * layers
        Ab = synthetic.activations(1, self.a_elems, seed + 100,
                                   dtype=synthetic.BF16 if bf16 else synthetic.F16)
        self.A_host = torch.from_numpy(Ab.view(np.int16).reshape(-1)).view(tdt).pin_memory()
        self.A = self.A_host.to(dev)
        self.C = torch.empty(self.c_elems, dtype=tdt, device=dev)
        self.C_host = torch.empty(self.c_elems, dtype=tdt).pin_memory()
        ws = max(native.w4a16_workspace_bytes(M, N, K, GROUP) for (_, K, N) in linears)
        self.ws = torch.zeros(max(ws, 16), dtype=torch.uint8, device=dev)
        # views per GEMM
        self.calls = []
        ao = co = 0
        for lay in self.layers:
            for w in lay:
                K, N = w["K"], w["N"]
                self.calls.append((w, self.A[ao:ao + M * K].view(M, K), self.C[co:co + M * N].view(M, N)))
                ao += M * K
                co += M * N
        self.bytes_per_step = sum(algorithmic_bytes(M, w["K"], w["N"]) for (w, _, _) in self.calls)
        self.weight_bytes = sum(w["weight_bytes"] for (w, _, _) in self.calls)

    def gemm(self, w, A, C):
        nat = self.native
        if self.tiled:
            nat.w4a16_gemm(A, w["tiled"], None, None, w["N"], GROUP, SYM, layout=nat.LAYOUT_TILED,
                           C=C, workspace=self.ws)
        else:
            nat.w4a16_gemm(A, w["codes"], w["scales"], w["zeros"], w["N"], GROUP, SYM, C=C,
                           workspace=self.ws)

    def step(self):
        for (w, A, C) in self.calls:
            self.gemm(w, A, C)


def tiled_supported(torch, native, qw, M=1):
    """Whether the library runs the tiled layout for M rows (probed with one call)."""
    K, N, codes, scales, zeros = qw
    try:
        t = native.w4a16_repack(codes, scales, zeros, K, N, GROUP, SYM)
        A = torch.zeros((M, K), dtype=torch.float16, device=codes.device)
        native.w4a16_gemm(A, t, None, None, N, GROUP, SYM, layout=native.LAYOUT_TILED)
        torch.cuda.synchronize()
        return True
    except native.W4A16Error as e:
        if e.status == native.EUNSUPPORTED:
            return False
        raise


def count_graph_kernels(graph):
    """Kernel nodes in a captured CUDA graph, through the driver API (None when unavailable)."""
    try:
        import ctypes

        cu = ctypes.CDLL("libcuda.so.1")
        raw = graph.raw_cuda_graph()
        handle = ctypes.c_void_p(int(raw))
        n = ctypes.c_size_t(0)
        if cu.cuGraphGetNodes(handle, None, ctypes.byref(n)) != 0:
            return None
        nodes = (ctypes.c_void_p * n.value)()
        if cu.cuGraphGetNodes(handle, nodes, ctypes.byref(n)) != 0:
            return None
        count = 0
        for i in range(n.value):
            t = ctypes.c_int(-1)
            if cu.cuGraphNodeGetType(ctypes.c_void_p(nodes[i]), ctypes.byref(t)) != 0:
                return None
            count += int(t.value == 0)  # CU_GRAPH_NODE_TYPE_KERNEL
        return count
    except Exception:
        return None


def new_graph(torch):
    """A torch CUDA graph that keeps its cudaGraph_t after instantiation (for node counting)."""
    try:
        return torch.cuda.CUDAGraph(keep_graph=True)
    except TypeError:
        return torch.cuda.CUDAGraph()


def time_graph(torch, graph, steps, world, dev):
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    torch.cuda.synchronize()
    start.record()
    for _ in range(steps):
        graph.replay()
    end.record()
    torch.cuda.synchronize()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    return start.elapsed_time(end) / steps


def time_per_launch(torch, stack, steps):
    """Per-GEMM device durations (CUDA events on the launching stream) for `steps` steps.
    A long sleep kernel first lets the host queue the launches ahead, so the events bracket
    device execution only. Returns {shape name: [ms, ...]}."""
    stream = torch.cuda.current_stream()
    out = {}
    for _ in range(steps):
        evs = []
        torch.cuda._sleep(int(60e6))
        for (w, A, C) in stack.calls:
            s = torch.cuda.Event(enable_timing=True)
            e = torch.cuda.Event(enable_timing=True)
            s.record(stream)
            stack.gemm(w, A, C)
            e.record(stream)
            evs.append((w["name"], w["K"], w["N"], s, e))
        torch.cuda.synchronize()
        for (name, K, N, s, e) in evs:
            out.setdefault((name, K, N), []).append(s.elapsed_time(e))
    return out


def time_e2e(torch, stack, steps, warmup):
    """The step through the public Python API, inputs from pinned host memory, outputs read
    back to pinned host memory every step; CUDA events around the whole step."""
    for _ in range(warmup):
        stack.A.copy_(stack.A_host, non_blocking=True)
        stack.step()
        stack.C_host.copy_(stack.C, non_blocking=True)
    torch.cuda.synchronize()
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record()
    for _ in range(steps):
        stack.A.copy_(stack.A_host, non_blocking=True)
        stack.step()
        stack.C_host.copy_(stack.C, non_blocking=True)
    end.record()
    torch.cuda.synchronize()
    return start.elapsed_time(end) / steps


def decode_sources_sha():
    """Hash of the decode kernel's sources (the files its ncu traffic capture depends on)."""
    import hashlib

    h = hashlib.sha256()
    for name in DECODE_SOURCES:
        with open(os.path.join(ROOT, "weight_only_int4_07_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def decode_traffic(bytes_per_launch):
    """DRAM bytes (read + write) per launch of the decode kernel from the committed ncu capture,
    scaled from the captured launch to `bytes_per_launch` algorithmic bytes (the kernel streams each
    unit record once, so its traffic grows with the units a launch processes). Returns
    (bytes or None, provenance); None when the kernel's sources changed after the capture."""
    if not os.path.exists(TRAFFIC_FILE):
        return None, None
    t = json.load(open(TRAFFIC_FILE))
    if t.get("sources_sha") != decode_sources_sha():
        return None, {"stale": True, "capture": t.get("capture")}
    ratio = t["dram_bytes"] / t["algorithmic_bytes"]
    return ratio * bytes_per_launch, {"ratio_to_algorithmic": ratio, "capture": t["capture"],
                                      "summary": t.get("summary")}


def time_stack(torch, native, synthetic, seed, layers, linears, bf16, steps, warmup, world, dev,
               gpu_index, e2e=True):
    """One decode step over a stack of linears (M = 1), replayed from a CUDA graph: device time per
    step (max over ranks), the kernel launches in the step, each shape's isolated launch time and,
    optionally, the end-to-end step through the Python API."""
    stack = DecodeStack(torch, native, synthetic, seed, layers=layers, linears=linears, bf16=bf16)
    torch.cuda.synchronize()
    for _ in range(max(warmup, 1)):
        stack.step()
    torch.cuda.synchronize()
    graph = new_graph(torch)
    with torch.cuda.graph(graph):
        stack.step()
    torch.cuda.synchronize()
    kernels_per_step = count_graph_kernels(graph)
    if hasattr(graph, "instantiate"):
        try:
            graph.instantiate()
        except RuntimeError:
            pass
    for _ in range(warmup):
        graph.replay()
    torch.cuda.synchronize()
    with ClockSampler(gpu_index) as clk:
        ms = time_graph(torch, graph, steps, world, dev)
    ms_max = max_over_ranks(ms, world, dev)
    launches = time_per_launch(torch, stack, 1)
    per_shape = {name: {"K": K, "N": N, "mean_us": 1e3 * statistics.mean(v),
                        "gbs": algorithmic_bytes(1, K, N) / (statistics.mean(v) * 1e-3) / 1e9}
                 for (name, K, N), v in launches.items()}
    out = {"ms_per_step": ms_max, "bytes_per_step": stack.bytes_per_step,
           "weight_bytes_per_step": stack.weight_bytes, "gemms_per_step": len(stack.calls),
           "kernels_per_step": kernels_per_step, "isolated_per_shape": per_shape,
           "clocks": clk.summary(), "tiled": stack.tiled}
    if e2e:
        e2e_ms = max_over_ranks(time_e2e(torch, stack, steps, warmup), world, dev)
        out["e2e"] = {"value": world * stack.bytes_per_step / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                      "h2d_bytes_per_step": stack.A.numel() * 2, "d2h_bytes_per_step": stack.C.numel() * 2,
                      "ms_per_step": e2e_ms}
    del graph, stack
    torch.cuda.synchronize()
    torch.cuda.empty_cache()
    return out


def bench_m256(torch, native, synthetic, seed, steps, warmup, copies=4):
    """TFLOPS of the (8192, 28672) sweep layer at M = 256, bf16 activations, rotating `copies`
    distinct weight copies (122 MB each) so that L2 cannot serve repeats."""
    dev = torch.device("cuda")
    K, N, M = SWEEP_K, SWEEP_N, SWEEP_M
    Wb = synthetic.weights_outliers(K, N, seed)
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).to(dev)
    codes, scales, zeros = native.w4a16_quantize(W, GROUP, SYM)
    del W
    use_tiled = tiled_supported(torch, native, (K, N, codes, scales, zeros), M)
    ws_need = native.w4a16_workspace_bytes(M, N, K, GROUP)
    ws = torch.zeros(max(ws_need, 16), dtype=torch.uint8, device=dev)
    if use_tiled:
        mats = [(None, None, None, native.w4a16_repack(codes, scales, zeros, K, N, GROUP, SYM))
                for _ in range(copies)]
    else:
        mats = [(codes.clone(), scales.clone(), zeros.clone(), None) for _ in range(copies)]
    del codes, scales, zeros
    Ab = synthetic.activations(M, K, seed + 1, dtype=synthetic.BF16)
    A = torch.from_numpy(Ab.view(np.int16)).view(torch.bfloat16).to(dev)
    C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)

    def run(i):
        c, s, z, t = mats[i % copies]
        if t is not None:
            native.w4a16_gemm(A, t, None, None, N, GROUP, SYM, layout=native.LAYOUT_TILED, C=C,
                              workspace=ws)
        else:
            native.w4a16_gemm(A, c, s, z, N, GROUP, SYM, C=C, workspace=ws)

    for i in range(warmup):
        run(i)
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()
    durs = []
    torch.cuda._sleep(int(20e6))
    evs = []
    for i in range(steps * copies):
        s = torch.cuda.Event(enable_timing=True)
        e = torch.cuda.Event(enable_timing=True)
        s.record(stream)
        run(i)
        e.record(stream)
        evs.append((s, e))
    torch.cuda.synchronize()
    durs = [s.elapsed_time(e) for (s, e) in evs]
    ms = statistics.mean(durs)
    kernel = native.w4a16_select_kernel(M, N, K, GROUP) if use_tiled else native.KERNEL_GEMV
    return {"M": M, "K": K, "N": N, "ms": ms, "tflops": gemm_flops(M, K, N) / (ms * 1e-3) / 1e12,
            "kernel": {1: "gemv", 2: "tc"}.get(kernel, str(kernel)), "dtype": "bf16",
            "bytes": algorithmic_bytes(M, K, N), "launches": len(durs),
            "layout": "tiled" if use_tiled else "plain"}


def bench_naive(torch, native, synthetic, seed, steps, warmup, copies=4):
    """The naive path the fused kernels are measured against: the packed weight expanded to a
    16-bit matrix by the library's dequantize kernel, then the library GEMM (torch.matmul, FP32
    accumulation). Per shape (the four Llama-3-8B decode linears at M = 1 with fp16 activations,
    and the sweep layer at M = 256 with bf16 activations) the mean device time of each half,
    rotating `copies` packed weight copies. GB/s counts the same algorithmic bytes as the fused
    path, so the two are directly comparable."""
    dev = torch.device("cuda")
    prev = (torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction,
            torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction)
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    shapes = [(name, K, N, 1, torch.float16, synthetic.F16) for (name, K, N) in LLAMA8B_LINEARS]
    shapes.append(("sweep_m256", SWEEP_K, SWEEP_N, SWEEP_M, torch.bfloat16, synthetic.BF16))
    stream = torch.cuda.current_stream()
    out = {}
    try:
        for i, (name, K, N, M, tdt, sdt) in enumerate(shapes):
            Wb = synthetic.weights_normal(K, N, seed + i)
            W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).to(dev)
            codes, scales, zeros = native.w4a16_quantize(W, GROUP, SYM)
            del W
            mats = [(codes.clone(), scales.clone(), None if zeros is None else zeros.clone())
                    for _ in range(copies)]
            del codes, scales, zeros
            Ab = synthetic.activations(M, K, seed + 50 + i, dtype=sdt)
            A = torch.from_numpy(Ab.view(np.int16)).view(tdt).to(dev)
            Wd = torch.empty((K, N), dtype=tdt, device=dev)
            C = torch.empty((M, N), dtype=tdt, device=dev)

            def run(j, evs=None):
                c, sc, z = mats[j % copies]
                if evs:
                    evs[0].record(stream)
                native.w4a16_dequantize(c, sc, z, K, N, GROUP, SYM, out=Wd)
                if evs:
                    evs[1].record(stream)
                torch.matmul(A, Wd, out=C)
                if evs:
                    evs[2].record(stream)

            for j in range(max(warmup, 1)):
                run(j)
            torch.cuda.synchronize()
            torch.cuda._sleep(int(20e6))
            rec = []
            for j in range(steps * copies):
                evs = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
                run(j, evs)
                rec.append(evs)
            torch.cuda.synchronize()
            deq = statistics.mean(e[0].elapsed_time(e[1]) for e in rec)
            mm = statistics.mean(e[1].elapsed_time(e[2]) for e in rec)
            tot = deq + mm
            out[name] = {"K": K, "N": N, "M": M, "acts": "fp16" if tdt == torch.float16 else "bf16",
                         "dequant_us": 1e3 * deq, "gemm_us": 1e3 * mm, "total_us": 1e3 * tot,
                         "gbs": algorithmic_bytes(M, K, N) / (tot * 1e-3) / 1e9,
                         "tflops": gemm_flops(M, K, N) / (tot * 1e-3) / 1e12,
                         "dequant_gbs": (algorithmic_bytes(0, K, N, out_bytes=0) + 2 * K * N)
                         / (deq * 1e-3) / 1e9}
            del mats, A, Wd, C
            torch.cuda.empty_cache()
    finally:
        (torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction,
         torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction) = prev
    return out


def bench_encoders(torch, native, synthetic, seed, reps=2, S=512, shapes=("qkv", "o", "gate_up", "down")):
    """The calibrated encoders (offline, once per layer), GPTQ and AWQ, on the Llama-3-8B decode
    shapes with S calibration rows (fp16): device time per layer (CUDA events around the whole
    call), and the layer-output error on the calibration inputs relative to RTN's, ||X W - X' W_hat||^2
    (X' = X for GPTQ, X S^-1 for AWQ)."""
    dev = torch.device("cuda")
    out = {}
    stream = torch.cuda.current_stream()
    for i, (name, K, N) in enumerate(LLAMA8B_LINEARS):
        if name not in shapes:
            continue
        W = torch.from_numpy(synthetic.weights_normal(K, N, seed + i).view(np.int16)).view(torch.float16).to(dev)
        X = torch.from_numpy(synthetic.calibration(S, K, seed + 50 + i).view(np.int16)).view(torch.float16).to(dev)
        ws = torch.empty(native.w4a16_gptq_workspace_bytes(K, N), dtype=torch.uint8, device=dev)
        q = native.w4a16_gptq_quantize(W, X, GROUP, SYM, workspace=ws)   # warm-up
        torch.cuda.synchronize()
        ms = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            q = native.w4a16_gptq_quantize(W, X, GROUP, SYM, workspace=ws)
            e1.record(stream)
            torch.cuda.synchronize()
            ms.append(e0.elapsed_time(e1))
        r = native.w4a16_quantize(W, GROUP, SYM)
        X64, W64 = X.double(), W.double()

        def err(qq):
            What = native.w4a16_dequantize(qq[0], qq[1], qq[2], K, N, GROUP, SYM).double()
            return float(((X64 @ (W64 - What)) ** 2).sum())

        # AWQ on the same layer: the encoded S W with inputs divided by s
        wsa = torch.empty(native.w4a16_awq_workspace_bytes(K, N, S), dtype=torch.uint8, device=dev)
        a = native.w4a16_awq_quantize(W, X, GROUP, SYM, workspace=wsa)   # warm-up
        torch.cuda.synchronize()
        ms_awq = []
        for _ in range(reps):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(stream)
            a = native.w4a16_awq_quantize(W, X, GROUP, SYM, workspace=wsa)
            e1.record(stream)
            torch.cuda.synchronize()
            ms_awq.append(e0.elapsed_time(e1))
        Da = native.w4a16_dequantize(a[0], a[1], a[2], K, N, GROUP, SYM).double()
        e_awq = float(((X64 @ W64 - (X64 / a[3].double()) @ Da) ** 2).sum())
        e_rtn = err(r)
        out[name] = {"K": K, "N": N, "calib_rows": S, "gptq_ms": statistics.mean(ms),
                     "gptq_output_error_vs_rtn": err(q) / e_rtn, "awq_ms": statistics.mean(ms_awq),
                     "awq_output_error_vs_rtn": e_awq / e_rtn}
        del W, X, ws, wsa, q, r, a, Da, X64, W64
        torch.cuda.empty_cache()
    return out


def bench_crossover(torch, native, synthetic, seed, Ms=SWEEP_MS, reps=6):
    """W4A16 against the W8A8 FP8 path on the (8192, 28672) sweep layer, bf16 activations, per
    batch size M: device time of one W4A16 GEMM (the library's dispatch on the tiled layout) and of
    one FP8 step (per-row activation quantization + the kind::f8f6f4 GEMM), each on two rotating
    weight copies (244 MB and 470 MB), and the smallest M where the FP8 step is faster -- the
    crossover of the pages' roofline argument."""
    dev = torch.device("cuda")
    K, N = SWEEP_K, SWEEP_N
    W = torch.from_numpy(synthetic.weights_outliers(K, N, seed).view(np.int16)).view(torch.float16).to(dev)
    codes, scales, zeros = native.w4a16_quantize(W, GROUP, SYM)
    tiled = [native.w4a16_repack(codes, scales, zeros, K, N, GROUP, SYM) for _ in range(2)]
    f8 = [native.w4a16_fp8_quantize_weights(W) for _ in range(2)]
    del W, codes, scales, zeros
    stream = torch.cuda.current_stream()
    out = []
    for M in Ms:
        A = torch.from_numpy(synthetic.activations(M, K, seed + M, dtype=synthetic.BF16).view(np.int16)).view(
            torch.bfloat16).to(dev)
        C = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
        ws = torch.zeros(max(native.w4a16_workspace_bytes(M, N, K, GROUP), 16), dtype=torch.uint8, device=dev)
        Aq = torch.empty((M, K), dtype=torch.uint8, device=dev)
        sa = torch.empty(M, dtype=torch.float32, device=dev)

        def w4(i):
            native.w4a16_gemm(A, tiled[i % 2], None, None, N, GROUP, SYM, layout=native.LAYOUT_TILED, C=C,
                              workspace=ws)

        def w8(i, quant=True):
            if quant:
                native.w4a16_fp8_quantize_acts(A, Aq, sa)
            native.w4a16_fp8_gemm(Aq, sa, f8[i % 2][0], f8[i % 2][1], C=C)

        res = {}
        for name, fn in (("w4a16", w4), ("fp8_step", w8), ("fp8_gemm", lambda i: w8(i, quant=False))):
            for i in range(3):
                fn(i)
            torch.cuda.synchronize()
            torch.cuda._sleep(int(20e6))
            evs = []
            for i in range(reps):
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                fn(i)
                e1.record(stream)
                evs.append((e0, e1))
            torch.cuda.synchronize()
            res[name] = statistics.mean(e0.elapsed_time(e1) for e0, e1 in evs) * 1e3
        flops = gemm_flops(M, K, N)
        out.append({"M": M, "w4a16_us": res["w4a16"], "fp8_step_us": res["fp8_step"],
                    "fp8_gemm_us": res["fp8_gemm"], "w4a16_tflops": flops / (res["w4a16"] * 1e-6) / 1e12,
                    "fp8_step_tflops": flops / (res["fp8_step"] * 1e-6) / 1e12})
        del A, C, ws, Aq, sa
    faster = [r["M"] for r in out if r["fp8_step_us"] < r["w4a16_us"]]
    del tiled, f8
    torch.cuda.empty_cache()
    return {"layer": {"K": K, "N": N, "acts": "bf16"}, "points": out,
            "crossover_M": (min(faster) if faster else None)}


def bench_variants(torch, native, synthetic, seed, copies=4, reps=6):
    """The format variants: K = N = 8192, weights 0.02 * Student-t(5), symmetric and asymmetric,
    group 32 and 128, fp16 and bf16 activations, M in {1, 16, 256}. Per variant the fused GEMM
    (the library's dispatch on the tiled layout) and the naive path (dequantize to 16 bits, then
    torch.matmul), mean device time over `copies` rotating weight copies (4 x 34-39 MB, more than
    L2 holds)."""
    dev = torch.device("cuda")
    K = N = 8192
    stream = torch.cuda.current_stream()
    prev = torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction, \
        torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction
    torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction = False
    torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction = False
    W = torch.from_numpy(synthetic.weights_student_t(K, N, seed).view(np.int16)).view(torch.float16).to(dev)
    out = []
    try:
        for sym in (1, 0):
            for group in (32, 128):
                codes, scales, zeros = native.w4a16_quantize(W, group, sym)
                tiled = [native.w4a16_repack(codes, scales, zeros, K, N, group, sym) for _ in range(copies)]
                for bf16 in (False, True):
                    tdt = torch.bfloat16 if bf16 else torch.float16
                    Wd = torch.empty((K, N), dtype=tdt, device=dev)
                    for M in (1, 16, 256):
                        A = torch.from_numpy(synthetic.activations(
                            M, K, seed + M, dtype=synthetic.BF16 if bf16 else synthetic.F16).view(np.int16)).view(
                            tdt).to(dev)
                        C = torch.empty((M, N), dtype=tdt, device=dev)
                        ws = torch.zeros(max(native.w4a16_workspace_bytes(M, N, K, group), 16), dtype=torch.uint8,
                                         device=dev)

                        def fused(i):
                            native.w4a16_gemm(A, tiled[i % copies], None, None, N, group, sym,
                                              layout=native.LAYOUT_TILED, C=C, workspace=ws)

                        def naive(i):
                            native.w4a16_dequantize(codes, scales, zeros, K, N, group, sym, out=Wd)
                            torch.matmul(A, Wd, out=C)

                        res = {}
                        for name, fn in (("fused", fused), ("naive", naive)):
                            for i in range(3):
                                fn(i)
                            torch.cuda.synchronize()
                            torch.cuda._sleep(int(20e6))
                            evs = []
                            for i in range(reps):
                                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                                e0.record(stream)
                                fn(i)
                                e1.record(stream)
                                evs.append((e0, e1))
                            torch.cuda.synchronize()
                            res[name] = statistics.mean(a.elapsed_time(b) for a, b in evs) * 1e3
                        nbytes = algorithmic_bytes(M, K, N, group=group, sym=sym)
                        out.append({"sym": bool(sym), "group": group, "acts": "bf16" if bf16 else "fp16", "M": M,
                                    "fused_us": res["fused"], "naive_us": res["naive"],
                                    "fused_gbs": nbytes / (res["fused"] * 1e-6) / 1e9,
                                    "fused_tflops": gemm_flops(M, K, N) / (res["fused"] * 1e-6) / 1e12,
                                    "kernel": {1: "gemv", 2: "tc"}.get(native.w4a16_select_kernel(M, N, K, group))})
                        del A, C, ws
                    del Wd
                del codes, scales, zeros, tiled
                torch.cuda.empty_cache()
    finally:
        (torch.backends.cuda.matmul.allow_fp16_reduced_precision_reduction,
         torch.backends.cuda.matmul.allow_bf16_reduced_precision_reduction) = prev
    del W
    torch.cuda.empty_cache()
    return {"K": K, "N": N, "weights": "0.02 * Student-t(5)", "points": out}


# ----------------------------------------------------------------------------- CPU oracle
def host_cores():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


ORACLE_COLS = 2048   # output columns of each 70B linear in the oracle's timed sample


def oracle_prepare(synthetic, seed, threads, linears=LLAMA70B_LINEARS, cols=ORACLE_COLS, a_dtype=1):
    """The oracle's timed sample of the headline workload: each linear of one Llama-3-70B-shaped
    layer restricted to its first `cols` output columns (RTN quantization is per column, so the
    sample has the layer's per-weight work), quantized by the oracle, one bf16 activation row."""
    import oracle

    packed = []
    for i, (name, K, N) in enumerate(linears):
        n = min(N, cols)
        Wb = synthetic.weights_normal(K, n, seed + i)
        st, c, s, z = oracle.quantize(Wb, GROUP, SYM, nthreads=threads)
        Ab = synthetic.activations(1, K, seed + 200 + i, dtype=a_dtype)
        packed.append((K, n, c, s, z, Ab, a_dtype))
    return packed


def oracle_pass(packed, threads):
    """One pass of the FP64 oracle over the sample's linears (M = 1, all sampled columns).
    Returns (algorithmic bytes, seconds)."""
    import oracle

    nbytes, secs = 0, 0.0
    for (K, N, c, s, z, Ab, a_dtype) in packed:
        t0 = time.perf_counter()
        oracle.linear(Ab, a_dtype, c, s, z, N, GROUP, SYM, nthreads=threads)
        secs += time.perf_counter() - t0
        nbytes += algorithmic_bytes(1, K, N)
    return nbytes, secs


def oracle_sample(synthetic, seed, threads, budget_s=15.0, packed=None):
    """The oracle's throughput, passes repeated while under the time budget (inputs prepared
    once, or reused from `packed`). Returns (GB/s, seconds, passes, packed)."""
    if packed is None:
        packed = oracle_prepare(synthetic, seed, threads)
    reps, total, nbytes = 0, 0.0, 0
    while reps < 1 or total < budget_s:
        b, t = oracle_pass(packed, threads)
        nbytes += b
        total += t
        reps += 1
    return nbytes / total / 1e9, total, reps, packed


ORACLE_SAMPLE = ("the four linears of one Llama-3-70B-shaped layer (8192x10240, 8192x8192, 8192x57344, "
                 "28672x8192), first %d output columns of each, M=1, g128 asym, bf16 acts; FP64 oracle" % ORACLE_COLS)


def oracle_configs(synthetic, threads, sub_cols=512):
    """The FP64 oracle (quantize excluded, the layer's matmul timed) on every configuration:
    full for the tiny layer and the Llama-3-8B linears; on the first `sub_cols` output columns of
    each layer for the sweep, the format variants and the 70B stack, extrapolated by the column
    count (the oracle's work is the same for every column) and labelled so."""
    import oracle

    def one(K, N, M, group, sym, a_dtype, seed, wfn=synthetic.weights_normal, cols=None):
        n = N if cols is None else min(N, cols)
        Wb = wfn(K, n, seed)
        _, c, s, z = oracle.quantize(Wb, group, sym, nthreads=threads)
        Ab = synthetic.activations(M, K, seed + 1, dtype=a_dtype)
        t0 = time.perf_counter()
        oracle.linear(Ab, a_dtype, c, s, z, n, group, sym, nthreads=threads)
        return (time.perf_counter() - t0) * N / n

    out = {"cores": threads, "unit": "s per GEMM"}
    out["tiny"] = {"M": 1, "K": 512, "N": 256, "s": one(512, 256, 1, 128, 0, 0, 1)}
    out["llama3_8b"] = {name: {"K": K, "N": N, "M": 1, "s": one(K, N, 1, GROUP, SYM, 0, 10 + i)}
                        for i, (name, K, N) in enumerate(LLAMA8B_LINEARS)}
    sweep = []
    for M in SWEEP_MS:
        t = one(SWEEP_K, SWEEP_N, M, GROUP, SYM, 1, 30, wfn=synthetic.weights_outliers, cols=sub_cols)
        sweep.append({"M": M, "s": t, "tflops": gemm_flops(M, SWEEP_K, SWEEP_N) / t / 1e12})
    out["sweep"] = {"K": SWEEP_K, "N": SWEEP_N, "points": sweep,
                    "extrapolated": f"from the first {sub_cols} of {SWEEP_N} columns"}
    var = []
    for sym in (1, 0):
        for group in (32, 128):
            for a_dtype in (0, 1):
                for M in (1, 16, 256):
                    var.append({"sym": bool(sym), "group": group, "acts": "bf16" if a_dtype else "fp16", "M": M,
                                "s": one(8192, 8192, M, group, sym, a_dtype, 40, wfn=synthetic.weights_student_t,
                                         cols=sub_cols)})
    out["variants"] = {"K": 8192, "N": 8192, "points": var,
                       "extrapolated": f"from the first {sub_cols} of 8192 columns"}
    stack = {}
    for M in (1, 8, 16):
        t = sum(one(K, N, M, GROUP, SYM, 1, 50 + i, cols=sub_cols) for i, (_, K, N) in enumerate(LLAMA70B_LINEARS))
        stack[str(M)] = {"s_per_step": t * LAYERS_70B}
    out["llama3_70b_stack"] = {"layers": LAYERS_70B, "per_M": stack,
                               "extrapolated": f"one layer, first {sub_cols} columns of each linear, x{LAYERS_70B} layers"}
    return out


# ----------------------------------------------------------------------------- arms
HEADLINE_WORKLOAD = ("llama3-70b decode linears (qkv 8192x10240, o 8192x8192, gate+up 8192x57344, "
                     "down 28672x8192), M=1, g128 asym INT4, bf16 acts, 80 layers per step")


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return 0
    from weight_only_int4_07_b200 import synthetic

    threads = host_cores()
    packed = oracle_prepare(synthetic, 11, threads)
    for _ in range(args.warmup):
        oracle_pass(packed, threads)
    tot_b, tot_s = 0, 0.0
    for _ in range(args.steps):
        b, t = oracle_pass(packed, threads)
        tot_b += b
        tot_s += t
    value = tot_b / tot_s / 1e9
    ms = 1e3 * tot_s / args.steps
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": HEADLINE_WORKLOAD, "sample_per_step": ORACLE_SAMPLE},
            "cpu_baseline": {"value": value, "unit": "GB/s", "cores": threads, "kind": "oracle",
                             "sample": ORACLE_SAMPLE + ", one pass per step"},
            "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args):
    import torch

    from weight_only_int4_07_b200 import build, native, synthetic

    rank, world, local_rank = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    if rank == 0:
        build.build()
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
    native.lib()
    peaks = load_peaks()

    # the headline: one decode step over the 70B-shaped stack
    r = time_stack(torch, native, synthetic, replica_seed(7000, rank), LAYERS_70B, LLAMA70B_LINEARS, True,
                   args.steps, args.warmup, world, dev, local_rank)
    ms_max = r["ms_per_step"]
    value = world * r["bytes_per_step"] / (ms_max * 1e-3) / 1e9
    # every launch of the step is the decode kernel (M = 1 on the tiled layout), so its mean
    # in-step duration is the step's device time over its launches
    n_launch = r["gemms_per_step"]
    kernel = native.w4a16_select_kernel(1, 8192, 8192, GROUP) if r["tiled"] else native.KERNEL_GEMV
    bytes_per_launch = r["bytes_per_step"] / n_launch
    launch_us = 1e3 * ms_max / n_launch
    achieved = bytes_per_launch / (launch_us * 1e-6) / 1e9
    traffic, traffic_src = decode_traffic(bytes_per_launch) if r["tiled"] else (None, None)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic,
                "kernel": "gemv_stream_kernel" if kernel == native.KERNEL_GEMV and r["tiled"] else
                {1: "gemv", 2: "tc"}.get(kernel, str(kernel)),
                "bytes_per_launch": bytes_per_launch, "launch_us_in_step": launch_us,
                "launches_per_step": n_launch, "peak_source": peaks["source"] + " (copy)",
                "traffic_source": traffic_src, "isolated_per_shape": r["isolated_per_shape"]}

    # the 32-layer Llama-3-8B stack (the smaller decode configuration)
    m1_8b = None
    if not args.skip_8b:
        r8 = time_stack(torch, native, synthetic, replica_seed(1000, rank), LAYERS, LLAMA8B_LINEARS, False,
                        args.steps, args.warmup, world, dev, local_rank, e2e=False)
        gbs8 = world * r8["bytes_per_step"] / (r8["ms_per_step"] * 1e-3) / 1e9
        m1_8b = {"value": gbs8, "unit": "GB/s", "ms_per_step": r8["ms_per_step"],
                 "frac": gbs8 / world / peaks["hbm_gbs"], "peak": peaks["hbm_gbs"],
                 "isolated_per_shape": r8["isolated_per_shape"], "clocks": r8["clocks"],
                 "config": {"workload": "llama3-8b decode linears (qkv 4096x6144, o 4096x4096, gate+up "
                                        "4096x28672, down 14336x4096), M=1, g128 asym INT4, fp16 acts, "
                                        "32 layers per step",
                            "gemms_per_step": r8["gemms_per_step"],
                            "algorithmic_bytes_per_step": r8["bytes_per_step"]}}

    # M = 256 on the sweep layer (TFLOPS)
    m256 = None
    if not args.skip_m256:
        rm = bench_m256(torch, native, synthetic, replica_seed(5000, rank), max(2, min(args.steps, 10)),
                        args.warmup)
        ms256 = max_over_ranks(rm["ms"], world, dev)
        tf = gemm_flops(rm["M"], rm["K"], rm["N"]) / (ms256 * 1e-3) / 1e12
        peak_tf = peaks["bf16_tflops"]
        m256 = {"value": world * tf, "unit": "TFLOP/s", "ms": ms256, "kernel": rm["kernel"],
                "roofline": {"bound": "tensor", "achieved": tf, "peak": peak_tf, "unit": "TFLOP/s",
                             "frac": tf / peak_tf, "traffic": None,
                             "peak_source": peaks["source"] + " burst"},
                "config": {"M": rm["M"], "K": rm["K"], "N": rm["N"], "group": GROUP, "sym": False,
                           "acts": "bf16", "weights": "N(0,0.02) with 0.1% outliers x20",
                           "l2": "4 rotating weight copies of 122 MB"}}

    naive = None
    if not args.skip_naive:
        naive = bench_naive(torch, native, synthetic, replica_seed(9000, rank), max(2, min(args.steps, 10)),
                            args.warmup)
        fused = dict(m1_8b["isolated_per_shape"]) if m1_8b else {}
        for name, rr in naive.items():
            us = (fused[name]["mean_us"] if name in fused
                  else (1e3 * m256["ms"] if (name == "sweep_m256" and m256) else None))
            rr["fused_us"] = us
            rr["fused_speedup"] = None if us is None else rr["total_us"] / us

    encoders = None
    if not args.skip_encoders:
        encoders = bench_encoders(torch, native, synthetic, replica_seed(9500, rank))

    crossover = None
    if not args.skip_crossover:
        crossover = bench_crossover(torch, native, synthetic, replica_seed(9700, rank))

    variants = None
    if not args.skip_variants:
        variants = bench_variants(torch, native, synthetic, replica_seed(9800, rank))

    cpu = None
    oracle_all = None
    if rank == 0 and world == 1 and not args.skip_cpu:
        threads = host_cores()
        gbs, secs, reps, packed = oracle_sample(synthetic, 11, threads, budget_s=args.cpu_budget)
        cpu = {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle",
               "sample": f"{reps} pass(es) over " + ORACLE_SAMPLE + f", {secs:.1f} s"}
        gbs1, secs1, _, _ = oracle_sample(synthetic, 11, 1, budget_s=0.0, packed=packed)
        cpu["single_thread"] = {"value": gbs1, "unit": "GB/s", "cores": 1, "seconds": secs1}
        if not args.skip_oracle_configs:
            oracle_all = oracle_configs(synthetic, threads)

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
                "data": "synthetic (seeded; weights N(0,0.02) fp16, activations N(0,1) bf16)",
                "config": {"workload": HEADLINE_WORKLOAD, "layers": LAYERS_70B,
                           "gemms_per_step": r["gemms_per_step"],
                           "weight_bytes_per_step": r["weight_bytes_per_step"],
                           "algorithmic_bytes_per_step": r["bytes_per_step"],
                           "parallelism": f"replica x{world}", "layout": "tiled" if r["tiled"] else "plain",
                           "l2": "inputs larger than L2: 35.6 GB of packed weights per step",
                           "timing": "CUDA graph replay of one step, CUDA events"},
                "e2e": r["e2e"], "roofline": roofline, "cpu_baseline": cpu, "clocks": r["clocks"],
                "gpu_launches": (None if r["kernels_per_step"] is None else r["kernels_per_step"] * args.steps),
                "m1_8b": m1_8b, "m256": m256, "naive": naive, "encoders": encoders,
                "crossover": crossover, "variants": variants, "oracle_configs": oracle_all}
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    return 0


def run_single(args):
    """A few launches of one tiled W4A16 GEMM (the small case profiled under ncu): weights of
    (K, N) on two rotating copies, M rows of activations; prints one line, times nothing."""
    import torch

    from weight_only_int4_07_b200 import build, native, synthetic

    K, N, M = (int(x) for x in args.single.split(","))
    torch.cuda.set_device(0)
    build.build()
    bf16 = args.dtype == "bf16"
    Wb = synthetic.weights_normal(K, N, 3)
    W = torch.from_numpy(Wb.view(np.int16)).view(torch.float16).cuda()
    codes, scales, zeros = native.w4a16_quantize(W, GROUP, SYM)
    del W
    copies = [native.w4a16_repack(codes, scales, zeros, K, N, GROUP, SYM) for _ in range(2)]
    Ab = synthetic.activations(M, K, 4, dtype=synthetic.BF16 if bf16 else synthetic.F16)
    A = torch.from_numpy(Ab.view(np.int16)).view(torch.bfloat16 if bf16 else torch.float16).cuda()
    C = torch.empty((M, N), dtype=A.dtype, device="cuda")
    ws = torch.zeros(max(native.w4a16_workspace_bytes(M, N, K, GROUP), 16), dtype=torch.uint8, device="cuda")
    for i in range(args.launches):
        native.w4a16_gemm(A, copies[i % 2], None, None, N, GROUP, SYM, layout=native.LAYOUT_TILED, C=C,
                          workspace=ws)
    torch.cuda.synchronize()
    print(json.dumps({"single": [K, N, M], "dtype": args.dtype, "launches": args.launches,
                      "kernel": {1: "gemv", 2: "tc"}[native.w4a16_select_kernel(M, N, K, GROUP)]}))
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--skip-m256", action="store_true")
    ap.add_argument("--skip-8b", action="store_true")
    ap.add_argument("--skip-variants", action="store_true")
    ap.add_argument("--skip-oracle-configs", action="store_true")
    ap.add_argument("--skip-cpu", action="store_true")
    ap.add_argument("--skip-naive", action="store_true")
    ap.add_argument("--skip-encoders", action="store_true")
    ap.add_argument("--skip-crossover", action="store_true")
    ap.add_argument("--cpu-budget", type=float, default=12.0)
    ap.add_argument("--single", default=None, help="K,N,M: a few launches of one GEMM, untimed")
    ap.add_argument("--dtype", choices=("f16", "bf16"), default="f16")
    ap.add_argument("--launches", type=int, default=4)
    args = ap.parse_args(argv)
    if args.single:
        return run_single(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
