"""Benchmark of the FP8 block-scaled NT GEMM on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--shapes auto|none|NAME,NAME,...] [--impl ours|reference]

One step = one call of the hot path (scheduling, TMA loads, tcgen05 MMA,
per-K-block promotion, epilogue; swap-AB and split-K for small M) on one
batch of seeded synthetic inputs already resident in HBM.  The headline
workload is the largest configuration of the method's benchmark set, the
M-grouped contiguous MoE-prefill GEMM (4 experts, 32768 tokens, N=4096,
K=7168).  A default run then times every configuration of that set (dense
128x256x512, dense decode M=64 and M=128 at N=2112 K=7168, dense
4096x7168x16384, the contiguous prefill, masked decode with 16 experts) with
the same steps, warm-up and L2 flush, and reports each under ``shapes`` with
its roofline fraction.  The ``quant_*`` workloads time the per-token 1x128
activation quantiser instead (GB/s of BF16 in + E4M3 and scales out).

L2 is flushed before every timed step (a 512 MB write, then a 256 MB read so
that no dirty line of the flush is left to write back during the step) and the
step is timed alone with CUDA events on the launching stream.  The end-to-end
figure (key ``e2e``) uploads every step's inputs from pinned host memory and
reads its result back, with the uploads, calls and downloads of consecutive
steps overlapped on three streams, as a serving loop would.  The masked GEMM
workloads are also timed as 50 calls replayed from one CUDA graph (key
``graph``).  SM clocks and throttle reasons are sampled through NVML while
every timed region runs.  Multi-GPU (torchrun): each rank runs its own
independent problem (no collective on the data path, weak scaling); every
time is the max over ranks.  ``--impl reference`` times the CPU oracle (FP64,
all host cores) on a bounded sample of the same workload instead.

Prints ONE JSON line on rank 0.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "FP8 TFLOPS and HBM GB/s per shape, % of B200 FP8/HBM roofline, 1 GPU"
# the largest configuration of the benchmark set: the headline of every run
DEFAULT_WORKLOAD = "contiguous_g4"
# the configurations of the method's benchmark set (DeepGEMM page 2 "性能实测"
# shapes plus the expert counts of the workload definitions), timed under
# ``shapes`` in every default run
SHAPES = ("dense_tiny", "dense_decode_m64", "dense_decode_m128", "dense_large", "contiguous_g4",
          "masked_g16")
# The pages' own figure for exactly the same workload (H800, another machine:
# context only).  DeepGEMM page 2 "性能实测": M=64 N=2112 K=7168 -> 1688 GB/s.
# The page's other rows leave one of M, N or K unstated, so no other workload
# has an exact counterpart.
PAGES_NUMBER = {"dense_decode_m64": (1688.0, "GB/s")}
# DRAM bytes per launch from ncu captures, keyed by kernel and workload, each
# with the hash of the kernel sources it was taken on
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
UNIT = {"dense_tiny": "TFLOP/s", "dense_decode_m64": "GB/s", "dense_decode_m128": "GB/s",
        "dense_large": "TFLOP/s", "contiguous_g4": "TFLOP/s", "masked_g16": "GB/s",
        "kgrouped_g4": "TFLOP/s",
        "bf16_dense_large": "TFLOP/s", "bf16_contiguous_g4": "TFLOP/s", "bf16_masked_g16": "GB/s",
        "bf16_dense_decode_m64": "GB/s", "ffn_g4": "TFLOP/s",
        "quant_tiny": "GB/s", "quant_tokens_32768": "GB/s", "quant_masked_g16": "GB/s"}
# the kernel each workload times, and the sources whose hash keys its ncu summary
KERNEL_SOURCES = {
    "fp8_gemm_kernel": ["moe_grouped_gemm_fp32_b200/csrc/gemm_kernel.cuh",
                        "moe_grouped_gemm_fp32_b200/csrc/ptx.cuh",
                        "moe_grouped_gemm_fp32_b200/csrc/dg_api.cu"],
    "quant_1x128_kernel": ["moe_grouped_gemm_fp32_b200/csrc/quant_kernel.cuh",
                           "moe_grouped_gemm_fp32_b200/csrc/quant_api.cu"],
    "bf16_gemm_kernel": ["moe_grouped_gemm_fp32_b200/csrc/bf16_kernel.cuh",
                         "moe_grouped_gemm_fp32_b200/csrc/bf16_api.cu",
                         "moe_grouped_gemm_fp32_b200/csrc/gemm_kernel.cuh",
                         "moe_grouped_gemm_fp32_b200/csrc/ptx.cuh"],
}
FLUSH_BYTES = 512 << 20
# B200 data-sheet figures, printed beside the measured denominators: HBM3e
# GB/s (HGX B200) and dense (no 2:4 sparsity) tensor TFLOP/s
NOMINAL_PEAK = {"hbm": 7700.0, "fp8": 4500.0, "bf16": 2250.0}
# masked decode calls are also timed replayed from one CUDA graph of this many
# back-to-back launches (the masked layout exists so that decode can be captured)
GRAPH_CALLS = 50
# Decode-sized workloads (inputs of 4 to 32 MB) are also timed as calls replayed
# back to back from one CUDA graph that cycles over copies of their inputs, as
# many as together exceed twice the L2 (126 MB): every call still reads its
# inputs from HBM, while the per-launch cost of an isolated, event-bracketed call
# after an L2 flush is left out.  The figure is the kernel's own duration plus
# the graph's launch gap between kernels.
L2_BYTES = 126 * 10**6
ROTATE_MIN_BYTES, ROTATE_MAX_BYTES = 4 << 20, 32 << 20


def rotation_sets(input_bytes: int) -> int:
    """Copies of a call's inputs for the rotating-graph timing (0: not timed)."""
    if not ROTATE_MIN_BYTES <= input_bytes <= ROTATE_MAX_BYTES:
        return 0
    return -(-2 * L2_BYTES // input_bytes) + 1


def is_quant(workload: str) -> bool:
    return workload.startswith("quant_")


def is_bf16(workload: str) -> bool:
    return workload.startswith("bf16_")


def kernel_name(workload: str) -> str:
    if is_quant(workload):
        return "quant_1x128_kernel"
    return "bf16_gemm_kernel" if is_bf16(workload) else "fp8_gemm_kernel"


def kernel_source_hash(kernel: str = "fp8_gemm_kernel") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as fh:
            return json.load(fh), "measured"
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}, "fallback"


def profiled_traffic(workload: str):
    """DRAM bytes per launch (ncu ``dram__bytes_read.sum + dram__bytes_write.sum``)
    of this workload's kernel from ``profiles/traffic.json``, or None when there
    is no capture or the kernel sources changed since it was taken."""
    kernel = kernel_name(workload)
    try:
        with open(TRAFFIC_FILE) as fh:
            entry = json.load(fh)["captures"][f"{kernel}/{workload}"]
    except (OSError, KeyError, ValueError):
        return None
    if entry.get("kernel_source_hash") != kernel_source_hash(kernel):
        return None
    return float(entry["dram_bytes_per_launch"])


class ClockSampler:
    """SM clock and throttle reasons of one GPU, read through NVML every
    millisecond by a background thread while a timed region runs (``resume`` /
    ``pause`` bracket each region; the samples of all regions are pooled).
    Reads only; no setting of the GPU is touched."""

    REASONS = (("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"))

    def __init__(self, torch_device):
        self.dev = torch_device
        self.samples = []
        self.stop_evt = threading.Event()
        self.active = threading.Event()
        self.thread = None
        self.nvml = None
        self.handle = None
        self.max_mhz = None

    def start(self):
        try:
            import pynvml
            import torch
            pynvml.nvmlInit()
            props = torch.cuda.get_device_properties(self.dev)
            bus = f"{props.pci_domain_id:08x}:{props.pci_bus_id:02x}:{props.pci_device_id:02x}.0"
            self.handle = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.handle, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
        except Exception:
            self.nvml = None
            return
        self.thread = threading.Thread(target=self._run, daemon=True)
        self.thread.start()

    def resume(self):
        self.active.set()

    def pause(self):
        self.active.clear()

    def _run(self):
        nv = self.nvml
        while not self.stop_evt.is_set():
            if not self.active.wait(0.05):
                continue
            try:
                mhz = nv.nvmlDeviceGetClockInfo(self.handle, nv.NVML_CLOCK_SM)
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.handle)
                if self.active.is_set():
                    self.samples.append((time.perf_counter(), mhz, mask))
            except Exception:
                pass
            self.stop_evt.wait(0.001)

    def stop(self):
        if self.thread is None:
            return None
        self.stop_evt.set()
        self.active.set()
        self.thread.join(timeout=5)
        if not self.samples:
            return None
        nv = self.nvml
        reasons = sorted({name for _, _, mask in self.samples for name, attr in self.REASONS
                          if mask & getattr(nv, attr, 0)})
        return {"sm_mhz": statistics.median(m for _, m, _ in self.samples),
                "sm_max_mhz": self.max_mhz, "reasons": reasons, "samples": len(self.samples)}


# ----------------------------------------------------------------------------- multi-rank plumbing
def rank_problem(workload: str, rank: int):
    """The problem rank `rank` times: the named workload for rank 0, and for
    other ranks the same shapes drawn from another seed (independent
    problems, weak scaling; no data moves between ranks)."""
    import workloads as W
    if is_quant(workload):
        return W.make_quant_workload(workload, seed_offset=7919 * rank)
    if is_bf16(workload):
        return W.make_bf16_workload(workload, seed_offset=7919 * rank)
    if workload in W.FFN_WORKLOADS:
        return W.make_ffn_workload(workload, seed_offset=7919 * rank)
    if rank == 0:
        return W.make_workload(workload)
    spec = dict(W.WORKLOADS[workload])
    spec["seed"] = spec["seed"] + 7919 * rank
    kind = spec.pop("kind")
    if kind == "dense":
        return W.make_dense(**spec)
    if kind == "contiguous":
        return W.make_contiguous_multinomial(spec["G"], spec["tokens"], spec["N"], spec["K"], spec["seed"])
    if kind == "k_grouped":
        return W.make_k_grouped_multinomial(spec["G"], spec["tokens"], spec["M"], spec["N"], spec["seed"])
    return W.make_masked_uniform(spec["G"], spec["Mmax"], spec["N"], spec["K"], spec["seed"])


def max_over_ranks(values, device, world: int):
    """Element-wise maximum of per-rank timings over all ranks (one small
    all-reduce on the control path; nothing else crosses ranks)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


# ----------------------------------------------------------------------------- our arm
class GemmCall:
    """Pinned host inputs, device output and the library call of one GEMM problem."""

    launches_per_step = 1
    OUT = ("d",)          # device outputs (each with a pinned host copy named <name>_host)

    def __init__(self, prob, dev):
        import numpy as np
        import torch
        self.prob = prob
        self.host = {k: torch.from_numpy(np.ascontiguousarray(v)).pin_memory()
                     for k, v in (("a", prob.a), ("sfa", prob.sfa), ("b", prob.b), ("sfb", prob.sfb))}
        if prob.m_indices is not None:
            self.host["m_indices"] = torch.from_numpy(prob.m_indices).pin_memory()
        if prob.masked_m is not None:
            self.host["masked_m"] = torch.from_numpy(prob.masked_m).pin_memory()
        if prob.ks is not None:
            self.host["ks"] = torch.from_numpy(prob.ks).pin_memory()
        self.d = torch.empty(prob.d_shape(), dtype=torch.bfloat16, device=dev)
        self.d_host = torch.empty(prob.d_shape(), dtype=torch.bfloat16).pin_memory()

    def call(self, t, stream):
        import moe_grouped_gemm_fp32_b200 as dg
        if self.prob.layout == "dense":
            dg.dg_fp8_gemm_nt(t["a"], t["sfa"], t["b"][0], t["sfb"][0], self.d, stream)
        elif self.prob.layout == "contiguous":
            dg.dg_m_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"], t["sfb"], self.d,
                                                   t["m_indices"], stream)
        elif self.prob.layout == "k_grouped":
            dg.dg_k_grouped_fp8_gemm_nt_contiguous(t["a"], t["sfa"], t["b"][0], t["sfb"][0], self.d,
                                                   t["ks"], stream)
        else:
            dg.dg_m_grouped_fp8_gemm_nt_masked(t["a"], t["sfa"], t["b"], t["sfb"], self.d,
                                               t["masked_m"], stream)

    def read_back(self):
        self.d_host.copy_(self.d, non_blocking=True)

    def d2h_bytes(self) -> int:
        return self.d.numel() * self.d.element_size()


class Bf16Call:
    """Pinned BF16 operands, device output and the library call of one BF16 GEMM."""

    launches_per_step = 1
    OUT = ("d",)

    def __init__(self, prob, dev):
        import numpy as np
        import torch
        self.prob = prob
        bf = lambda x: torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
        self.host = {"a": bf(prob.a).pin_memory(), "b": bf(prob.b).pin_memory()}
        if prob.m_indices is not None:
            self.host["m_indices"] = torch.from_numpy(prob.m_indices).pin_memory()
        if prob.masked_m is not None:
            self.host["masked_m"] = torch.from_numpy(prob.masked_m).pin_memory()
        self.d = torch.empty(prob.d_shape(), dtype=torch.bfloat16, device=dev)
        self.d_host = torch.empty(prob.d_shape(), dtype=torch.bfloat16).pin_memory()

    def call(self, t, stream):
        import moe_grouped_gemm_fp32_b200 as dg
        if self.prob.layout == "dense":
            dg.dg_bf16_gemm_nt(t["a"], t["b"][0], self.d, stream)
        elif self.prob.layout == "contiguous":
            dg.dg_m_grouped_bf16_gemm_nt_contiguous(t["a"], t["b"], self.d, t["m_indices"], stream)
        else:
            dg.dg_m_grouped_bf16_gemm_nt_masked(t["a"], t["b"], self.d, t["masked_m"], stream)

    def read_back(self):
        self.d_host.copy_(self.d, non_blocking=True)

    def d2h_bytes(self) -> int:
        return self.d.numel() * self.d.element_size()


class FFNCall:
    """Pinned tokens and expert weights, device intermediate and output, and the
    fused expert FFN call (two launches: GEMM1 + SwiGLU + requantisation, GEMM2)."""

    launches_per_step = 2
    OUT = ("y",)

    def __init__(self, prob, dev):
        import numpy as np
        import torch
        self.prob = prob
        t = lambda x: torch.from_numpy(np.ascontiguousarray(x)).pin_memory()
        self.host = {"a": t(prob.a), "sfa": t(prob.sfa), "w1": t(prob.w1), "sfb1": t(prob.sfb1),
                     "w2": t(prob.w2), "sfb2": t(prob.sfb2), "m_indices": t(prob.m_indices)}
        self.q = torch.empty((prob.M, prob.I), dtype=torch.uint8, device=dev)
        self.s = torch.empty((prob.I // 128, prob.ld_sfa), dtype=torch.float32, device=dev)
        self.y = torch.empty((prob.M, prob.H), dtype=torch.bfloat16, device=dev)
        self.y_host = torch.empty((prob.M, prob.H), dtype=torch.bfloat16).pin_memory()

    def call(self, t, stream):
        import moe_grouped_gemm_fp32_b200 as dg
        dg.dg_m_grouped_fp8_ffn_contiguous(t["a"], t["sfa"], t["w1"], t["sfb1"], t["w2"], t["sfb2"],
                                           self.q, self.s, self.y, t["m_indices"], stream)

    def read_back(self):
        self.y_host.copy_(self.y, non_blocking=True)

    def d2h_bytes(self) -> int:
        return self.y.numel() * self.y.element_size()


class QuantCall:
    """Pinned BF16 activations, device codes and scales, and the quantiser call."""

    launches_per_step = 1
    OUT = ("q", "sfa")

    def __init__(self, prob, dev):
        import torch
        self.prob = prob
        self.host = {"x": prob.x_bf16().pin_memory()}
        if prob.masked_m is not None:
            self.host["masked_m"] = torch.from_numpy(prob.masked_m).pin_memory()
        shape = tuple(prob.x.shape)
        sshape = (prob.KB, prob.ld_sfa) if prob.layout == "dense" else (prob.G, prob.KB, prob.ld_sfa)
        self.q = torch.empty(shape, dtype=torch.uint8, device=dev)
        self.sfa = torch.empty(sshape, dtype=torch.float32, device=dev)
        self.q_host = torch.empty(shape, dtype=torch.uint8).pin_memory()
        self.sfa_host = torch.empty(sshape, dtype=torch.float32).pin_memory()

    def call(self, t, stream):
        import moe_grouped_gemm_fp32_b200 as dg
        if self.prob.layout == "dense":
            dg.dg_per_token_cast_to_fp8(t["x"], self.q, self.sfa, stream)
        else:
            dg.dg_per_token_cast_to_fp8_masked(t["x"], self.q, self.sfa, t["masked_m"], stream)

    def read_back(self):
        self.q_host.copy_(self.q, non_blocking=True)
        self.sfa_host.copy_(self.sfa, non_blocking=True)

    def d2h_bytes(self) -> int:
        return self.q.numel() + self.sfa.numel() * 4

def make_call(workload: str, prob, dev):
    """The call object (pinned host inputs, device outputs, library call) of a workload."""
    if is_quant(workload):
        return QuantCall(prob, dev)
    if is_bf16(workload):
        return Bf16Call(prob, dev)
    return FFNCall(prob, dev) if prob.layout == "ffn_contiguous" else GemmCall(prob, dev)


@dataclasses.dataclass
class Timing:
    """Device timing of one workload: the mean and median step time (each the
    max over ranks) and the number of this library's kernels per step."""
    workload: str
    prob: object
    ms: float
    ms_median: float
    launches: int
    graph_ms: float = 0.0      # rotating-graph ms per call (decode-sized workloads), else 0
    graph_sets: int = 0
    graph_calls: int = 0


class DeviceBench:
    """The device side of one rank: L2 flush buffers, the launching stream, the
    barrier that brackets every timed region and the clock sampler."""

    def __init__(self, dev, world: int, local_rank: int):
        import torch
        self.dev, self.world, self.local_rank = dev, world, local_rank
        self.stream = torch.cuda.current_stream(dev)
        self.flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
        self.flush_read = torch.ones(FLUSH_BYTES // 8, dtype=torch.float32, device=dev)
        self.sampler = ClockSampler(dev)

    def flush_l2(self, i: int):
        # write > L2 (evicts every input line), then read > L2 so the dirty lines
        # of the write are written back now and the timed step starts from a
        # cold, clean L2
        self.flush.fill_(float(i))
        self.flush_read.sum()

    def barrier(self):
        import torch
        import torch.distributed as dist
        if self.world > 1:
            dist.barrier(device_ids=[self.local_rank])
        torch.cuda.synchronize(self.dev)

    def time_steps(self, step, steps: int, warmup: int):
        """W untimed warm-up steps, then exactly K steps, each after an L2 flush
        and timed alone with CUDA events on the launching stream; the region is
        bracketed by a barrier and a device synchronisation on both sides.
        Returns (mean ms, median ms), each the max over ranks."""
        import torch
        import moe_grouped_gemm_fp32_b200 as dg
        for i in range(warmup):
            self.flush_l2(i)
            step()
        dg.dg_get_device_status(clear=True)
        self.barrier()
        self.sampler.resume()
        starts = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        ends = [torch.cuda.Event(enable_timing=True) for _ in range(steps)]
        for i in range(steps):
            self.flush_l2(i)                      # every step starts from HBM
            starts[i].record(self.stream)
            step()
            ends[i].record(self.stream)
        self.barrier()
        self.sampler.pause()
        per_step = [a.elapsed_time(b) for a, b in zip(starts, ends)]
        status = dg.dg_get_device_status(clear=True)
        if status:
            raise RuntimeError(f"kernel status word {status:#x}")
        ms, med = max_over_ranks([sum(per_step) / len(per_step), statistics.median(per_step)],
                                 self.dev, self.world)
        return ms, med


def time_workload(bench: DeviceBench, workload: str, rank: int, steps: int, warmup: int,
                  keep: bool = False):
    """Device timing of one workload on this rank's problem; with ``keep`` also
    the call object and its device inputs (for the end-to-end and graph timings)."""
    prob = rank_problem(workload, rank)
    op = make_call(workload, prob, bench.dev)
    devt = {k: v.to(bench.dev, non_blocking=False) for k, v in op.host.items()}
    ms, med = bench.time_steps(lambda: op.call(devt, bench.stream), steps, warmup)
    t = Timing(workload, prob, ms, med, op.launches_per_step)
    sets = rotation_sets(sum(v.numel() * v.element_size() for v in op.host.values()))
    if sets and not is_quant(workload):
        t.graph_sets, t.graph_calls = sets, max(GRAPH_CALLS, 2 * sets)
        t.graph_ms = rotating_graph_ms(bench, op, sets, t.graph_calls)
    return (t, op, devt) if keep else t


def rotating_graph_ms(bench: DeviceBench, op, sets: int, calls: int, replays: int = 5) -> float:
    """Milliseconds per call: ``calls`` calls captured in one CUDA graph, call i
    reading input copy i % sets, replayed back to back (median of ``replays``
    replays, each timed with CUDA events on the launching stream; max over
    ranks).  No flush: the copies together exceed twice the L2."""
    import torch
    import moe_grouped_gemm_fp32_b200 as dg
    ins = [{k: v.to(bench.dev) for k, v in op.host.items()} for _ in range(sets)]
    side = torch.cuda.Stream(bench.dev)
    side.wait_stream(bench.stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for i in range(calls):
            op.call(ins[i % sets], side)
    bench.stream.wait_stream(side)
    g.replay()
    bench.barrier()
    bench.sampler.resume()
    times = []
    for _ in range(replays):
        st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        st.record(bench.stream)
        g.replay()
        en.record(bench.stream)
        torch.cuda.synchronize(bench.dev)
        times.append(st.elapsed_time(en) / calls)
    bench.sampler.pause()
    del g, ins
    bench.barrier()
    status = dg.dg_get_device_status(clear=True)
    if status:
        raise RuntimeError(f"kernel status word {status:#x}")
    return max_over_ranks([statistics.median(times)], bench.dev, bench.world)[0]


def e2e_pipelined(bench: DeviceBench, op, steps: int, warmup: int) -> float:
    """Milliseconds per step end to end, the way a serving loop runs it: every
    step uploads its inputs from pinned host memory, calls the library and reads
    its result back to pinned host memory.  Three streams pipeline consecutive
    steps (upload of step i+1, compute of step i, download of step i-1) over two
    sets of device inputs and outputs; the events that order them keep each set
    from being overwritten before its use ends.  The timed region runs from an
    event before the first upload to an event after the last download."""
    import torch
    dev, comp = bench.dev, bench.stream
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    host = op.host
    ins = [{k: v.to(dev) for k, v in host.items()} for _ in range(2)]
    outs = [{n: getattr(op, n) for n in op.OUT}, {n: torch.empty_like(getattr(op, n)) for n in op.OUT}]
    host_outs = [{n: getattr(op, n + "_host") for n in op.OUT},
                 {n: torch.empty_like(getattr(op, n + "_host")).pin_memory() for n in op.OUT}]
    ev = lambda: torch.cuda.Event()
    uploaded, computed, downloaded = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    for e in computed + downloaded:
        e.record(comp)

    def run(n):
        for i in range(n):
            j = i & 1
            s_in.wait_event(computed[j])              # step i-2 no longer reads input set j
            with torch.cuda.stream(s_in):
                for k, v in host.items():
                    ins[j][k].copy_(v, non_blocking=True)
            uploaded[j].record(s_in)
            comp.wait_event(uploaded[j])
            comp.wait_event(downloaded[j])            # step i-2's result has left output set j
            for name in op.OUT:
                setattr(op, name, outs[j][name])
            op.call(ins[j], comp)
            computed[j].record(comp)
            s_out.wait_event(computed[j])
            with torch.cuda.stream(s_out):
                for name in op.OUT:
                    host_outs[j][name].copy_(outs[j][name], non_blocking=True)
            downloaded[j].record(s_out)
        comp.wait_stream(s_in)
        comp.wait_stream(s_out)

    run(max(2, warmup // 2))
    bench.barrier()
    bench.sampler.resume()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    n = max(2, min(steps, 50))
    start.record(comp)
    s_in.wait_stream(comp)
    s_out.wait_stream(comp)
    run(n)
    end.record(comp)
    bench.barrier()
    bench.sampler.pause()
    for name in op.OUT:
        setattr(op, name, outs[0][name])
    return start.elapsed_time(end) / n


def launch_floor_ms(bench: DeviceBench, steps: int, warmup: int) -> float:
    """Event-timed step of an empty kernel (torch's zero-cycle sleep kernel)
    under the same flush and events: the timing method's own floor."""
    import torch
    ms, _ = bench.time_steps(lambda: torch.cuda._sleep(0), steps, warmup)
    return ms


def run_ours(args, rank, world, local_rank):
    """Times the headline workload (device-resident and end to end from pinned
    host buffers, plus the CUDA-graph replay for masked GEMMs), then every
    workload of ``shapes``.  Returns (headline Timing, e2e ms, h2d bytes, d2h
    bytes, graph ms, [Timing of each shape], clocks, launch-floor ms)."""
    import torch
    from moe_grouped_gemm_fp32_b200 import build as dg_build

    dg_build.build()
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    bench = DeviceBench(dev, world, local_rank)
    bench.sampler.start()

    # ---- the headline: device-resident timing
    head, op, devt = time_workload(bench, args.workload, rank, args.steps, args.warmup, keep=True)
    stream = bench.stream

    # ---- end to end through the public API from pinned host buffers
    e2e_ms = e2e_pipelined(bench, op, args.steps, args.warmup)
    host = op.host
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = op.d2h_bytes()

    graph_ms = 0.0
    if head.prob.layout == "masked" and not is_quant(args.workload):
        bench.sampler.resume()
        graph_ms = graph_timing(op, devt, dev, stream)
        bench.sampler.pause()
    import moe_grouped_gemm_fp32_b200 as dg
    status = dg.dg_get_device_status(clear=True)
    if status:
        raise RuntimeError(f"kernel status word {status:#x}")
    e2e_ms, graph_ms = max_over_ranks([e2e_ms, graph_ms], dev, world)
    del op, devt

    # ---- the other configurations of the benchmark set, same steps and flush
    shapes = []
    for w in args.shape_list:
        if w == args.workload:
            shapes.append(head)
            continue
        shapes.append(time_workload(bench, w, rank, args.steps, args.warmup))
        torch.cuda.empty_cache()
    floor_ms = launch_floor_ms(bench, args.steps, args.warmup) if args.shape_list else 0.0
    clocks = bench.sampler.stop()
    return head, e2e_ms, h2d, d2h, graph_ms, shapes, clocks, floor_ms


def graph_timing(op, devt, dev, stream, replays: int = 5) -> float:
    """Milliseconds per call with GRAPH_CALLS calls captured in one CUDA graph and
    replayed back to back (median of ``replays`` replays).  No L2 flush between
    the calls: the masked workloads' B operand alone is larger than L2, so B
    still streams from HBM on every call while A may stay in L2."""
    import torch
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        for _ in range(GRAPH_CALLS):
            op.call(devt, side)
    stream.wait_stream(side)
    g.replay()
    torch.cuda.synchronize(dev)
    times = []
    for _ in range(replays):
        st = torch.cuda.Event(enable_timing=True)
        en = torch.cuda.Event(enable_timing=True)
        st.record(stream)
        g.replay()
        en.record(stream)
        torch.cuda.synchronize(dev)
        times.append(st.elapsed_time(en) / GRAPH_CALLS)
    del g
    torch.cuda.synchronize(dev)
    return statistics.median(times)


def metric_value(prob, unit, ms, world):
    if unit == "GB/s":
        return prob.bytes() * world / (ms * 1e-3) / 1e9
    return prob.flops() * world / (ms * 1e-3) / 1e12


def quant_cpu_baseline(prob, budget_s=10.0):
    """The oracle quantiser as it stands (OpenMP over all host cores) on a
    bounded sample: evenly spaced valid rows, as many as fit ~budget_s,
    scaled linearly to the whole workload."""
    import numpy as np
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    if prob.layout == "dense":
        rows = prob.x
    else:
        rows = np.concatenate([prob.x[g, :int(prob.masked_m[g])] for g in range(prob.G)])
    n_all = rows.shape[0]
    t0 = time.perf_counter()
    oracle.quantize_1x128(rows[:min(n_all, 16)])
    per_row = (time.perf_counter() - t0) / max(1, min(n_all, 16))
    n = int(min(n_all, max(16, budget_s / max(per_row, 1e-9))))
    pick = rows[:: max(1, n_all // n)][:n]
    t0 = time.perf_counter()
    oracle.quantize_1x128(pick)
    dt = time.perf_counter() - t0
    secs = dt * n_all / len(pick)
    value = prob.bytes() / secs / 1e9
    return {"value": value, "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": f"{len(pick)} of {n_all} valid rows, {dt:.2f} s, scaled linearly to the whole workload",
            "seconds_per_step": secs}


def bf16_cpu_baseline(prob, unit, budget_s=10.0):
    """The oracle BF16 GEMM as it stands (FP64 accumulation, all host cores) on
    evenly spaced valid output rows, as many as fit ~budget_s, scaled linearly."""
    import numpy as np
    import oracle
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    if prob.layout == "masked":
        sel = [(g, m) for g in range(prob.G) for m in range(int(prob.masked_m[g]))]
    elif prob.layout == "contiguous":
        sel = [(int(prob.m_indices[m]), m) for m in np.flatnonzero(prob.m_indices >= 0)]
    else:
        sel = [(0, m) for m in range(prob.M)]

    def run(pick):
        # one dense call per group over its picked rows (OpenMP over the rows)
        for g in sorted({q[0] for q in pick}):
            rows = [m for gg, m in pick if gg == g]
            a = prob.a[g, rows] if prob.layout == "masked" else prob.a[rows]
            oracle.gemm_bf16("dense", a, prob.b[g], len(rows), prob.N, prob.K)
    probe = sel[:: max(1, len(sel) // 32)][:32]
    t0 = time.perf_counter()
    run(probe)
    per_row = (time.perf_counter() - t0) / len(probe)
    n = max(len(probe), min(len(sel), int(budget_s / max(per_row, 1e-9))))
    pick = sel[:: max(1, len(sel) // n)][:n]
    t0 = time.perf_counter()
    run(pick)
    dt = time.perf_counter() - t0
    secs = dt * len(sel) / len(pick)
    value = (prob.bytes() / secs / 1e9) if unit == "GB/s" else (prob.flops() / secs / 1e12)
    return {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
            "sample": f"{len(pick)} of {len(sel)} valid output rows (all N columns), {dt:.1f} s, "
                      f"scaled linearly to the whole workload", "seconds_per_step": secs}


def cpu_baseline(prob, unit, budget_s=10.0):
    """The oracle as it stands (FP64, OpenMP over all host cores) on a bounded
    sample: whole problems repeated until ~budget_s, or a leading slice of the
    output rows when one whole problem would take longer."""
    import numpy as np
    import oracle
    if not hasattr(prob, "flops"):
        return quant_cpu_baseline(prob, budget_s)
    if not hasattr(prob, "sfa"):
        return bf16_cpu_baseline(prob, unit, budget_s)
    if prob.layout == "ffn_contiguous":
        oracle.build()
        valid = np.flatnonzero(prob.m_indices >= 0)
        t0 = time.perf_counter()
        oracle.ffn_rows(prob, valid[:: max(1, len(valid) // 8)][:8])
        per_row = (time.perf_counter() - t0) / 8
        n = max(8, min(len(valid), int(budget_s / per_row)))
        pick = valid[:: max(1, len(valid) // n)][:n]
        t0 = time.perf_counter()
        oracle.ffn_rows(prob, pick)
        dt = time.perf_counter() - t0
        secs = dt * len(valid) / len(pick)
        return {"value": prob.flops() / secs / 1e12, "unit": unit, "cores": len(os.sched_getaffinity(0)),
                "kind": "oracle", "seconds_per_step": secs,
                "sample": f"{len(pick)} of {len(valid)} token rows through both GEMMs, {dt:.1f} s, "
                          f"scaled linearly to the whole workload"}
    oracle.build()
    cores = len(os.sched_getaffinity(0))
    t0 = time.perf_counter()
    probe_rows = max(1, min(prob.M, 8))
    if prob.layout == "k_grouped":
        # output rows are (group, row) pairs: G * M of them, each of N columns
        sel = [(g, m) for g in range(prob.G) for m in range(prob.M)]
        t0 = time.perf_counter()
        probe = sel[:: max(1, len(sel) // probe_rows)][:probe_rows]
        oracle.points(prob, np.repeat([q[0] for q in probe], prob.N), np.repeat([q[1] for q in probe], prob.N),
                      np.tile(np.arange(prob.N), len(probe)))
        per_row = (time.perf_counter() - t0) / len(probe)
        n_rows = max(1, min(len(sel), int(budget_s / per_row)))
        pick = sel[:: max(1, len(sel) // n_rows)][:n_rows]
        t0 = time.perf_counter()
        oracle.points(prob, np.repeat([q[0] for q in pick], prob.N), np.repeat([q[1] for q in pick], prob.N),
                      np.tile(np.arange(prob.N), len(pick)))
        dt = time.perf_counter() - t0
        secs = dt * len(sel) / len(pick)
        value = (prob.bytes() / secs / 1e9) if unit == "GB/s" else (prob.flops() / secs / 1e12)
        return {"value": value, "unit": unit, "cores": cores, "kind": "oracle",
                "sample": f"{len(pick)} of {len(sel)} (group, row) output rows (all N columns), {dt:.1f} s, "
                          f"scaled linearly to the whole workload", "seconds_per_step": secs}
    if prob.layout == "masked":
        g = int(np.argmax(prob.masked_m))
        rows = np.arange(min(probe_rows, int(prob.masked_m[g])))
        grp = np.full(len(rows) * prob.N, g)
    else:
        valid = np.flatnonzero(prob.m_indices >= 0) if prob.layout == "contiguous" else np.arange(prob.M)
        rows = valid[:probe_rows]
        grp = np.zeros(len(rows) * prob.N, np.int64)
    rr = np.repeat(rows, prob.N)
    cc = np.tile(np.arange(prob.N), len(rows))
    oracle.points(prob, grp, rr, cc)
    t_probe = time.perf_counter() - t0
    per_row = t_probe / len(rows)
    full_rows = prob.valid_rows()
    if per_row * full_rows <= budget_s:
        reps, t0 = 0, time.perf_counter()
        while True:
            oracle.solve(prob)
            reps += 1
            if time.perf_counter() - t0 >= budget_s:
                break
        secs = (time.perf_counter() - t0) / reps
        sample = f"{reps} full solve(s) of the workload, {secs:.3f} s each"
    else:
        n_rows = max(1, int(budget_s / per_row))
        if prob.layout == "masked":
            sel = [(g, r) for g in range(prob.G) for r in range(int(prob.masked_m[g]))]
            sel = sel[:: max(1, len(sel) // n_rows)][:n_rows]
            grp = np.repeat([s[0] for s in sel], prob.N)
            rr = np.repeat([s[1] for s in sel], prob.N)
        else:
            valid = np.flatnonzero(prob.m_indices >= 0) if prob.layout == "contiguous" else np.arange(prob.M)
            pick = valid[:: max(1, len(valid) // n_rows)][:n_rows]
            grp = np.zeros(len(pick) * prob.N, np.int64)
            rr = np.repeat(pick, prob.N)
        n_rows = len(rr) // prob.N
        cc = np.tile(np.arange(prob.N), n_rows)
        t0 = time.perf_counter()
        oracle.points(prob, grp, rr, cc)
        dt = time.perf_counter() - t0
        secs = dt * full_rows / n_rows
        sample = (f"{n_rows} of {full_rows} valid output rows (all N columns), "
                  f"{dt:.1f} s, scaled linearly to the whole workload")
    value = (prob.bytes() / secs / 1e9) if unit == "GB/s" else (prob.flops() / secs / 1e12)
    return {"value": value, "unit": unit, "cores": cores, "kind": "oracle", "sample": sample,
            "seconds_per_step": secs}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    prob = rank_problem(args.workload, 0)
    unit = UNIT[args.workload]
    # per-step CPU budget: the whole --steps/--warmup run stays within a few minutes
    budget = max(0.2, min(2.0, 120.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_baseline(prob, unit, budget_s=budget)
    vals = [cpu_baseline(prob, unit, budget_s=budget) for _ in range(args.steps)]
    secs = sum(v["seconds_per_step"] for v in vals) / len(vals)
    value = (prob.bytes() / secs / 1e9) if unit == "GB/s" else (prob.flops() / secs / 1e12)
    line = {"metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": secs * 1e3, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "f32" if is_quant(args.workload) else "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": args.workload, **shape_config(prob)},
            "cpu_baseline": {"value": value, "unit": unit, "cores": vals[0]["cores"],
                             "kind": "oracle", "sample": vals[0]["sample"]},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def shape_config(prob):
    if getattr(prob, "layout", "") == "ffn_contiguous":
        return {"layout": "contiguous expert FFN (GEMM1 + SwiGLU + requantise, GEMM2)", "G": prob.G,
                "M_total": prob.M, "valid_rows": prob.valid_rows(), "H": prob.H, "I": prob.I}
    if hasattr(prob, "flops") and not hasattr(prob, "sfa"):   # BF16 GEMM
        c = {"layout": prob.layout, "N": prob.N, "K": prob.K, "operands": "bf16"}
        if prob.layout == "dense":
            c["M"] = prob.M
        elif prob.layout == "contiguous":
            c.update(G=prob.G, M_total=prob.M, valid_rows=prob.valid_rows())
        else:
            c.update(G=prob.G, Mmax=prob.M, valid_rows=prob.valid_rows())
        return c
    if not hasattr(prob, "flops"):          # quantiser inputs
        c = {"layout": prob.layout, "K": prob.K, "in": "bf16", "out": "e4m3 + f32 1x128 scales"}
        if prob.layout == "dense":
            c["M"] = prob.M
        else:
            c.update(G=prob.G, Mmax=prob.M, valid_rows=prob.valid_rows())
        return c
    c = {"layout": prob.layout, "N": prob.N, "K": prob.K}
    if prob.layout == "dense":
        c["M"] = prob.M
    elif prob.layout == "contiguous":
        c.update(G=prob.G, M_total=prob.M, valid_rows=prob.valid_rows())
    elif prob.layout == "k_grouped":
        c.update(G=prob.G, M=prob.M, ks=[int(k) for k in prob.ks])
    else:
        c.update(G=prob.G, Mmax=prob.M, valid_rows=prob.valid_rows())
    return c


def roofline(workload: str, prob, ms: float):
    """Roofline entry of one workload's kernel: algorithmic bytes (HBM-bound) or
    FLOP (tensor-bound) per launch over the measured step time, against the
    measured peak, and the ncu DRAM traffic of one launch when it is current."""
    peaks, peak_src = measured_peaks()
    unit = UNIT[workload]
    if unit == "GB/s":
        bound, peak, runit = "hbm", peaks["hbm_gbs"], "GB/s"
        nominal = NOMINAL_PEAK["hbm"]
        achieved = prob.bytes() / (ms * 1e-3) / 1e9
        src = "hbm_gbs"
    else:
        bound, runit = "tensor", "TFLOP/s"
        # BF16: the measured BF16 peak; FP8 dense = 2 x BF16 dense (nominal ratio)
        peak = peaks["bf16_tflops"] * (1.0 if is_bf16(workload) else 2.0)
        nominal = NOMINAL_PEAK["bf16" if is_bf16(workload) else "fp8"]
        achieved = prob.flops() / (ms * 1e-3) / 1e12
        src = "bf16_tflops" if is_bf16(workload) else "2 x bf16_tflops"
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": runit, "frac": achieved / peak,
            "traffic": profiled_traffic(workload), "nominal_peak": nominal,
            "frac_of_nominal": achieved / nominal, "peak_source": f"{peak_src} ({src})"}


def shape_entry(t: Timing, world: int):
    unit = UNIT[t.workload]
    e = {"value": metric_value(t.prob, unit, t.ms, world), "unit": unit, "ms_per_step": t.ms,
         "ms_median": t.ms_median, "launches_per_step": t.launches,
         "roofline": roofline(t.workload, t.prob, t.ms), "config": shape_config(t.prob)}
    pages = PAGES_NUMBER.get(t.workload)
    if pages and pages[1] == unit:
        e["vs_pages"] = e["value"] / pages[0]
    if t.graph_ms > 0:
        g = {"value": metric_value(t.prob, unit, t.graph_ms, world), "unit": unit,
             "ms_per_call": t.graph_ms, "calls_per_graph": t.graph_calls, "input_copies": t.graph_sets,
             "l2": "not flushed: call i reads input copy i mod input_copies, the copies together "
                   "exceed twice the L2"}
        g["frac"] = roofline(t.workload, t.prob, t.graph_ms)["frac"]
        if pages and pages[1] == unit:
            g["vs_pages"] = g["value"] / pages[0]
        e["graph_rotating"] = g
    return e


def parse_shapes(arg: str, workload: str):
    if arg == "none":
        return []
    if arg == "auto":
        return list(SHAPES) if workload == DEFAULT_WORKLOAD else []
    names = [w for w in arg.split(",") if w]
    for w in names:
        if w not in UNIT:
            raise SystemExit(f"unknown workload {w!r}")
    return names


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--shapes", default="auto",
                    help="workloads timed after the headline under 'shapes': auto (the benchmark "
                         "set when the headline is the default workload), none, or a comma list")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload not in UNIT:
        ap.error(f"unknown workload {args.workload!r}")
    args.shape_list = parse_shapes(args.shapes, args.workload)

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import torch
    import torch.distributed as dist
    from datetime import timedelta
    if world > 1:
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=timedelta(seconds=300),
                                device_id=torch.device("cuda", local_rank))
    try:
        head, e2e_ms, h2d, d2h, graph_ms, shapes, clocks, floor_ms = run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            dist.destroy_process_group()
    if rank != 0:
        return 0
    prob, ms, unit = head.prob, head.ms, UNIT[args.workload]
    value = metric_value(prob, unit, ms, world)
    pages = PAGES_NUMBER.get(args.workload)
    measurement = {"l2": "flushed before every step (512 MB write, then 256 MB read)",
                   "gbps": prob.bytes() / (ms * 1e-3) / 1e9, "ms_median_step": head.ms_median}
    if not is_quant(args.workload):
        measurement["tflops"] = prob.flops() / (ms * 1e-3) / 1e12
    if floor_ms > 0:
        measurement["launch_floor_ms"] = floor_ms
        measurement["launch_floor"] = "an empty kernel timed the same way (flush, events around one launch)"
    line = {
        "metric": METRIC, "value": value, "unit": unit, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": (value / pages[0]) if pages and pages[1] == unit else None,
        "dtype": ("f32 (bf16 in, e4m3 out)" if is_quant(args.workload)
                  else "bf16 (f32 accumulate, bf16 out)" if is_bf16(args.workload)
                  else "e4m3 (f32 accumulate, bf16 out)"),
        "data": "synthetic",
        "config": {"workload": args.workload, **shape_config(prob)},
        "roofline": roofline(args.workload, prob, ms),
        "e2e": {"value": metric_value(prob, unit, e2e_ms, world), "unit": unit,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                "how": "pinned host inputs uploaded, library call, result read back, every step; "
                       "three streams overlap the upload of step i+1, the compute of step i and "
                       "the download of step i-1"},
        "gpu_launches": args.steps * head.launches,
        "clocks": clocks,
        "measurement": measurement,
    }
    if graph_ms > 0:
        line["graph"] = {"value": metric_value(prob, unit, graph_ms, world), "unit": unit,
                         "ms_per_call": graph_ms, "calls_per_graph": GRAPH_CALLS,
                         "l2": "not flushed between calls (B alone exceeds L2)"}
    if head.graph_ms > 0:
        line["graph_rotating"] = shape_entry(head, world)["graph_rotating"]
    if shapes:
        line["shapes"] = {t.workload: shape_entry(t, world) for t in shapes}
    if not args.no_cpu_baseline and world == 1:
        cb = cpu_baseline(prob, unit)
        cb.pop("seconds_per_step", None)
        line["cpu_baseline"] = cb
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
