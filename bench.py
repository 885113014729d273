#!/usr/bin/env python3
"""Benchmark of the LittleBit compressed-linear forward on B200.

One step = one forward pass of every layer of a synthetic Llama-2-shaped
stack (both binary contractions, all scalings, both paths) through the C ABI.
Default workload: the Llama-2-70B-shaped decode stack at ~0.1 BPW (560
layers, M = 1, 857 MB of packed signs and scales: larger than L2, so every
step streams from HBM).  The same JSON line carries the Llama-2-13B-shaped
prefill stack (M = 2048, tensor-core bound) as "prefill".

Metric: algorithmic bytes (packed signs + binary16 scales + x + y) per second
for decode, algorithmic FLOPs (2*M*2r*(K+N) per layer) per second for prefill.

The JSON line also carries: "roofline" (the dominant kernel against the
measured peak, with its full-size DRAM traffic while the kernel sources match
the capture in profiles/traffic.txt), "e2e" (the same step through the C ABI
from pinned host x to pinned host y, steps pipelined over two device buffer
sets; the serial figure beside it), "cpu_baseline" (the float64 oracle on a
bounded sample), "backward" (QAT backward of one Llama-2-13B-shaped block),
"init" (Dual-SVID + residual initialisation of one Llama-2-7B-shaped block, and
its LittleBit-2 variant with Joint-ITQ as "init.littlebit2"), clocks and
tokens/s.

Usage:  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
        python bench.py --impl reference ...   (the CPU oracle, timed as is)
Multi-GPU: one process per GPU (torchrun); every rank runs the whole stack
(independent replicas, weak scaling); time = max over ranks.
"""

from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from sub_bit_weight_b200 import synth  # noqa: E402

METRIC = "LittleBit linear decode GB/s & prefill TFLOP/s, % of B200 roofline"
DECODE_DEFAULT = "llama2_70b_0.1"
PREFILL_DEFAULT = "llama2_13b_0.3_prefill"
INIT_DEFAULT = "llama2_7b_0.1"
BACKWARD_DEFAULT = "llama2_13b_0.3_prefill"
# the other workloads, each at its batch sizes; the stack that fits in L2 both warm and with L2 flushed per step
CONFIGS_DEFAULT = ("single_512:1,single_512:8,llama2_7b_0.1:1,llama2_7b_0.1:1:flushed,"
                   "llama2_7b_0.55:1,llama2_7b_0.55:4,llama2_7b_0.55:16")
INIT_ITERS = 24
ITQ_ITERS = 50          # Joint-ITQ alternations of the LittleBit-2 initialisation (iterative quantisation's usual 50)
# binary64 FMA rate of B200: 148 SMs x 64 FP64 FMA per clock x 2 FLOP at the 1965 MHz maximum SM clock
FP64_PEAK_TFLOPS = 148 * 64 * 2 * 1.965e9 / 1e12


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "src": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "src": "fallback"}


# ----------------------------------------------------------------- measured DRAM traffic

CSRC = os.path.join(ROOT, "sub_bit_weight_b200", "csrc")
KERNEL_SOURCES = {
    "quantize_pair_kernel": ["lb_decode_pair.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "finish_pair_kernel": ["lb_decode_pair.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "contraction1_ldg_kernel": ["lb_decode_pair.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "contraction2_ldg_kernel": ["lb_decode_pair.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "contraction1_kernel": ["lb_decode.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "contraction2_kernel": ["lb_decode.cu", "lb_decode_common.cuh", "lb_internal.cuh"],
    "prefill_kernel<0>": ["lb_prefill.cu", "lb_prefill.cuh", "lb_prefill_types.cuh", "lb_tc.cuh", "lb_internal.cuh"],
    "prefill_kernel<1>": ["lb_prefill.cu", "lb_prefill.cuh", "lb_prefill_types.cuh", "lb_tc.cuh", "lb_internal.cuh"],
    "gemm_at_b_kernel": ["lb_gemm.cu", "lb_tc.cuh", "lb_internal.cuh"],
}


def source_hash(kernel: str) -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES.get(kernel, []):
        with open(os.path.join(CSRC, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def measured_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from profiles/traffic.txt, only while the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.txt")
    if not os.path.exists(path):
        return None
    want = source_hash(kernel)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == kernel and parts[1] == workload:
                return float(parts[3]) if parts[2] == want else None
    return None


def prefill_traffic(workload: str):
    """DRAM bytes of one prefill step (both tensor-core launches), while their sources are unchanged."""
    t = [measured_traffic(k, workload) for k in ("prefill_kernel<0>", "prefill_kernel<1>")]
    return None if any(v is None for v in t) else sum(t)


# ----------------------------------------------------------------- algorithmic work

def layer_bytes(s: synth.LayerShape, M: int, npaths: int = 2):
    """(contraction-1 bytes, contraction-2 bytes) of one layer: signs, scales, x, y."""
    k1 = npaths * (s.K * s.r / 8 + 2 * s.K + 2 * s.r) + 2 * M * s.K
    k2 = npaths * (s.N * s.r / 8 + 2 * s.N) + 4 * M * s.N
    return k1, k2


def layer_flops(s: synth.LayerShape, M: int, npaths: int = 2):
    return 2.0 * M * npaths * s.r * (s.K + s.N)


# ----------------------------------------------------------------- clocks

class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int, period: float = 0.005):
        self.samples, self.reasons = [], set()
        self.period = period
        self._stop = threading.Event()
        self.max_mhz = None
        self.nvml_index = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.nvml_index = self.nvml_index_of(pynvml, index)
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.nvml_index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # NVML missing: report that
            self.nv = None
            self.err = str(e)

    @staticmethod
    def nvml_index_of(nv, torch_index: int) -> int:
        """NVML index of CUDA device ``torch_index``: the NVML device with the same PCI domain, bus and device
        numbers (CUDA_VISIBLE_DEVICES renumbers the devices CUDA sees, not those NVML sees); the same index
        when no device matches or the lookup fails."""
        try:
            import torch
            p = torch.cuda.get_device_properties(torch_index)
            want = (int(p.pci_domain_id), int(p.pci_bus_id), int(p.pci_device_id))
            for i in range(nv.nvmlDeviceGetCount()):
                info = nv.nvmlDeviceGetPciInfo(nv.nvmlDeviceGetHandleByIndex(i))
                if (int(info.domain), int(info.bus), int(info.device)) == want:
                    return i
        except Exception:
            pass
        return torch_index

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for b, name in self.REASONS.items():
                    if bits & b and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.nv:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.nv:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "nvml_index": self.nvml_index}


# ----------------------------------------------------------------- CPU oracle baseline

def oracle_sample(w: synth.Workload, M: int, budget_s: float, max_layers: int | None = None):
    """Time the oracle (as it stands) on the first layers of the stack until the budget is used."""
    import oracle
    shapes = [s for _, s in w.layers()]
    done_bytes = done_flops = 0.0
    n = 0
    elapsed = 0.0
    pools = {}
    for idx, s in enumerate(shapes):
        inp = synth.layer_inputs(w.seed, idx, s)
        inp["U"] = [oracle.pack_signs(F) for F in inp.pop("F_U")]
        inp["V"] = [oracle.pack_signs(F) for F in inp.pop("F_V")]
        xb = synth.layer_activations(w, idx, M, s.K, pools)
        rows = M
        if w.pool_rows:             # prefill: a bounded number of activation rows
            rows = max(1, min(M, 4))
            xb = xb[:rows]
        t0 = time.perf_counter()
        oracle.forward(np.ascontiguousarray(xb), inp)
        elapsed += time.perf_counter() - t0
        b1, b2 = layer_bytes(s, rows)
        done_bytes += b1 + b2
        done_flops += layer_flops(s, rows)
        n += 1
        if elapsed >= budget_s or (max_layers and n >= max_layers):
            break
    return {"seconds": elapsed, "layers": n, "bytes": done_bytes, "flops": done_flops,
            "rows": rows if w.pool_rows else M}


# ----------------------------------------------------------------- GPU runs

def run_gpu(w: synth.Workload, M: int, steps: int, warmup: int, dist, dev, want_e2e=True, nblocks=None,
            flush_l2=False):
    import torch
    from sub_bit_weight_b200 import lib, stacks

    layers, shapes = stacks.build_workload(w, device=dev, nblocks=nblocks)
    S = lib.lb_stack_create(layers)
    # contiguous x / y so that the end-to-end run moves them with one copy each way
    xsz = [M * s.K for s in shapes]
    ysz = [M * s.N for s in shapes]
    x_all = torch.empty(sum(xsz), dtype=torch.bfloat16, device=dev)
    y_all = torch.empty(sum(ysz), dtype=torch.float32, device=dev)
    xs_src, _ = stacks.workload_activations(w, shapes, M, device=dev)
    xs, ys = [], []
    ox = oy = 0
    for s, a, b, src in zip(shapes, xsz, ysz, xs_src):
        xs.append(x_all[ox:ox + a].view(M, s.K))
        xs[-1].copy_(src)
        ys.append(y_all[oy:oy + b].view(M, s.N))
        ox += a
        oy += b
    del xs_src
    io = lib.StackIO(S, xs, ys)
    stream = torch.cuda.current_stream()

    for _ in range(warmup):
        lib.lb_stack_forward(S, io=io)
    torch.cuda.synchronize()
    nl = lib.lb_last_launch_count()

    nlaunch_per_step = None
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    # whole steps: no events between a step's launches (consecutive kernels may overlap)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.nvtx.range_push("bench_timed")       # lets a profiler select the timed launches
        if flush_l2:
            # a 256 MB write (twice the L2) before every step; only the steps are timed, each with its own events
            flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
            se = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
            for k in range(steps):
                flush.zero_()
                se[k][0].record(stream)
                lib.lb_stack_forward(S, io=io)
                se[k][1].record(stream)
                if nlaunch_per_step is None:
                    nlaunch_per_step = lib.lb_last_launch_count()
            torch.cuda.synchronize()
            total_ms = sum(a.elapsed_time(b) for a, b in se)
            del flush
        else:
            start.record(stream)
            for k in range(steps):
                lib.lb_stack_forward(S, io=io)
                if nlaunch_per_step is None:
                    nlaunch_per_step = lib.lb_last_launch_count()
            stop.record(stream)
            torch.cuda.synchronize()
            total_ms = start.elapsed_time(stop)
        torch.cuda.nvtx.range_pop()
    if dist:
        dist.barrier()

    # each kernel alone: a CUDA event after every launch (launches then run strictly one after another)
    pk_steps = max(3, min(steps, 100))
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(nl + 1)] for _ in range(pk_steps)]
    for trio in ev:          # torch creates the CUDA event on first record
        for e in trio:
            e.record(stream)
    torch.cuda.synchronize()
    for k in range(pk_steps):
        lib.lb_profile_events(ev[k])
        lib.lb_stack_forward(S, io=io)
    torch.cuda.synchronize()
    lib.lb_profile_events([])
    per_launch = None
    if nlaunch_per_step == nl and nl in (2, 3, 4):
        per_launch = tuple(sum(e[i].elapsed_time(e[i + 1]) for e in ev) / pk_steps for i in range(nl))

    e2e = None
    if want_e2e:
        hx = torch.empty(x_all.numel(), dtype=torch.bfloat16, pin_memory=True)
        hx.copy_(x_all)
        hy = torch.empty(y_all.numel(), dtype=torch.float32, pin_memory=True)
        e_steps = max(3, min(steps, 200))
        for _ in range(2):
            x_all.copy_(hx, non_blocking=True)
            lib.lb_stack_forward(S, io=io)
            hy.copy_(y_all, non_blocking=True)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(e_steps):
            x_all.copy_(hx, non_blocking=True)
            lib.lb_stack_forward(S, io=io)
            hy.copy_(y_all, non_blocking=True)
        b.record(stream)
        torch.cuda.synchronize()
        serial_ms = a.elapsed_time(b) / e_steps
        y_serial = hy.clone()
        # pipelined steps, as a serving loop runs them: two device x / y buffer sets and host y buffers; step i's
        # host->device copy (copy stream in) and step i-1's device->host copy (copy stream out) overlap step i's
        # compute; every step still copies its own inputs in and its whole result out inside the timed region
        xb, yb = [x_all, torch.empty_like(x_all)], [y_all, torch.empty_like(y_all)]
        hyb = [hy, torch.empty(y_all.numel(), dtype=torch.float32, pin_memory=True)]
        offs_x = [0] + [int(v) for v in np.cumsum(xsz)]
        offs_y = [0] + [int(v) for v in np.cumsum(ysz)]
        io2 = lib.StackIO(S, [xb[1][offs_x[i]:offs_x[i + 1]].view(M, s.K) for i, s in enumerate(shapes)],
                          [yb[1][offs_y[i]:offs_y[i + 1]].view(M, s.N) for i, s in enumerate(shapes)])
        ios = [io, io2]
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_c = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def piped(n):
            for i in range(n):
                k = i % 2
                if i >= 2:
                    s_in.wait_event(ev_c[k])           # step i-2's compute has read xb[k]
                with torch.cuda.stream(s_in):
                    xb[k].copy_(hx, non_blocking=True)
                ev_in[k].record(s_in)
                stream.wait_event(ev_in[k])
                if i >= 2:
                    stream.wait_event(ev_out[k])       # step i-2's result has left yb[k]
                lib.lb_stack_forward(S, io=ios[k], stream=stream)
                ev_c[k].record(stream)
                s_out.wait_event(ev_c[k])
                with torch.cuda.stream(s_out):
                    hyb[k].copy_(yb[k], non_blocking=True)
                ev_out[k].record(s_out)
            stream.wait_stream(s_out)

        piped(4)
        torch.cuda.synchronize()
        if dist:
            dist.barrier()
        a.record(stream)
        s_in.wait_stream(stream)
        piped(e_steps)
        b.record(stream)
        torch.cuda.synchronize()
        # the decode sums are exact (integer MMAs, float64 chunk sums): every step's result equals the serial one
        if not (torch.equal(hyb[0], y_serial) and torch.equal(hyb[1], y_serial)):
            raise RuntimeError("pipelined end-to-end steps produced different outputs")
        e2e = {"ms": a.elapsed_time(b) / e_steps, "h2d": x_all.numel() * 2, "d2h": y_all.numel() * 4,
               "steps": e_steps, "serial_ms": serial_ms}
    out = {"total_ms": total_ms, "per_launch": per_launch, "launches": nlaunch_per_step * steps,
           "clocks": clk.summary(), "e2e": e2e, "shapes": shapes}
    del S, layers, io
    torch.cuda.synchronize()
    return out


def max_over_ranks(v: float, dist):
    """The largest of every rank's v (a device time): one all-reduce, taken by every rank in the same order."""
    if not dist:
        return v
    import torch
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def replica_throughput(world: int, work_per_rank: float, steps: int, max_ms: float) -> float:
    """Whole-job throughput of independent replicas: every rank's work over the slowest rank's time."""
    return world * work_per_rank * steps / (max_ms * 1e-3)


def roofline_of(res: dict, shapes, M: int, prefill: bool, pk: dict, wkey: str):
    """Roofline object of the dominant kernel of one stack step, from the per-launch event timings of run_gpu.

    Decode: algorithmic bytes of the kernel (layer_bytes) over its average launch time, against measured HBM copy
    bandwidth.  Prefill: algorithmic FLOPs of the kernel over its launch time, against the measured bf16 tensor
    peak; each kernel is timed alone (an event on each side), so the burst figure is the denominator, with the
    sustained one beside it.
    """
    if not res["per_launch"]:
        return None
    if prefill:
        k1ms, k2ms = res["per_launch"][:2]
        dom = 1 if k2ms >= k1ms else 0
        f1 = sum(2.0 * M * 2 * s.r * s.K for s in shapes)
        f2 = sum(2.0 * M * 2 * s.r * s.N for s in shapes)
        dom_w, dom_ms = (f2, k2ms) if dom else (f1, k1ms)
        ach = dom_w / (dom_ms * 1e-3) / 1e12
        kname = "prefill_kernel<1>" if dom else "prefill_kernel<0>"
        return {"bound": "tensor", "kernel": kname + (" (output GEMM)" if dom else " (latent GEMM)"),
                "achieved": round(ach, 1), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
                "frac": round(ach / pk["bf16_tflops"], 4),
                "peak_src": pk["src"] + " bf16 burst (dense 16-bit tensor peak; the kernel is timed alone)",
                "frac_of_sustained": round(ach / pk["bf16_tflops_sustained"], 4),
                "traffic": measured_traffic(kname, wkey),
                "per_kernel_ms": {"latent": round(k1ms, 4), "output": round(k2ms, 4)},
                "per_kernel_flops": {"latent": f1, "output": f2},
                "per_kernel_tflops": {"latent": round(f1 / (k1ms * 1e-3) / 1e12, 1),
                                      "output": round(f2 / (k2ms * 1e-3) / 1e12, 1)}}
    k1b = sum(layer_bytes(s, M)[0] for s in shapes)
    k2b = sum(layer_bytes(s, M)[1] for s in shapes)
    suffix = "_ldg_kernel" if M <= 2 else "_kernel"
    names = ["contraction1" + suffix, "contraction2" + suffix]
    kbytes = [k1b, k2b]
    if len(res["per_launch"]) == 3:
        # general kernels (3..16 rows): the per-layer finish between the contractions moves no algorithmic bytes
        names = [names[0], "finish_general_kernel", names[1]]
        kbytes = [k1b, 0.0, k2b]
    if len(res["per_launch"]) == 4:
        # activation quantisation and the contraction-1 finish run as their own launches:
        # x and g are the bytes of the first, the finish moves no algorithmic bytes
        qb = sum(2.0 * M * s.K + 2 * 2.0 * s.K for s in shapes)
        names = ["quantize_pair_kernel", names[0], "finish_pair_kernel", names[1]]
        kbytes = [qb, k1b - qb, 0.0, k2b]
    kms = list(res["per_launch"])
    di = max(range(len(kms)), key=lambda i: kms[i])
    dom_bytes, dom_ms, kname = kbytes[di], kms[di], names[di]
    ach = dom_bytes / (dom_ms * 1e-3) / 1e9
    return {"bound": "hbm", "kernel": kname,
            "achieved": round(ach, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": round(ach / pk["hbm_gbs"], 4), "peak_src": pk["src"],
            "traffic": measured_traffic(kname, wkey), "algorithmic_bytes_per_launch": dom_bytes,
            "per_kernel_ms": {n: round(t, 5) for n, t in zip(names, kms)},
            "per_kernel_bytes": {n: b for n, b in zip(names, kbytes)}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DECODE_DEFAULT, choices=sorted(synth.WORKLOADS))
    ap.add_argument("--M", type=int, default=None)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--prefill", default=PREFILL_DEFAULT, help="prefill workload for the 'prefill' object ('' = skip)")
    ap.add_argument("--prefill-steps", type=int, default=5)
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--blocks", type=int, default=None, help="only the first N blocks of the stack (profiling)")
    ap.add_argument("--flush-l2", action="store_true",
                    help="write 256 MB before every timed step and time the steps alone (stacks that fit in L2)")
    ap.add_argument("--init", default=INIT_DEFAULT,
                    help="workload whose first block gets the Dual-SVID + residual initialisation ('' = skip)")
    ap.add_argument("--init-steps", type=int, default=2)
    ap.add_argument("--init-warmup", type=int, default=3)
    ap.add_argument("--init-layers", default="", help="comma-separated layer names of the block (default: all)")
    ap.add_argument("--backward", default=BACKWARD_DEFAULT,
                    help="workload whose first block gets the QAT backward pass ('' = skip)")
    ap.add_argument("--backward-steps", type=int, default=5)
    ap.add_argument("--configs", default=CONFIGS_DEFAULT,
                    help="comma-separated workload[:M[:flushed]] runs for the 'configs' object ('' = skip)")
    ap.add_argument("--config-steps", type=int, default=200)
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.gpus != world:
        # one process per GPU: N > 1 ranks come from the launcher, never from this flag alone
        sys.stderr.write(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}; run N ranks as "
                         f"python -m torch.distributed.run --nproc-per-node N bench.py --gpus N\n")
        sys.exit(2)
    w = synth.WORKLOADS[args.workload]
    M = args.M if args.M is not None else w.Ms[0]
    pk = peaks()

    if args.impl == "reference":
        return reference_arm(args, w, M, world, rank, pk)

    import torch
    dist = None
    if world > 1:
        import torch.distributed as tdist
        local = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(local)
        import datetime
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    dev = torch.device("cuda", torch.cuda.current_device())

    res = run_gpu(w, M, args.steps, args.warmup, dist, dev, nblocks=args.blocks, want_e2e=not w.pool_rows,
                  flush_l2=args.flush_l2)
    total_ms = max_over_ranks(res["total_ms"], dist)
    shapes = res["shapes"]
    ms_step = total_ms / args.steps
    prefill_main = bool(w.pool_rows)
    if prefill_main:
        flops = sum(layer_flops(s, M) for s in shapes)
        value = replica_throughput(world, flops, args.steps, total_ms) / 1e12
        unit = "TFLOP/s"
    else:
        k1b = sum(layer_bytes(s, M)[0] for s in shapes)
        k2b = sum(layer_bytes(s, M)[1] for s in shapes)
        step_bytes = k1b + k2b
        value = replica_throughput(world, step_bytes, args.steps, total_ms) / 1e9
        unit = "GB/s"

    roof = roofline_of(res, shapes, M, prefill_main, pk, w.key)
    e2e = e2e_of(res, dist, world, flops if prefill_main else step_bytes, prefill_main,
                 "lb_stack_forward from pinned host x to pinned host y")
    line = {"metric": METRIC, "value": round(value, 2), "unit": unit, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": ("bf16 in, fp16 tcgen05 MMA (fp32 accumulate in TMEM), fp32 out" if prefill_main else
                      "bf16 in, int8 tensor-core MMA (u8 signs x s8 fixed-point digits, s32 acc), fp32 out"),
            "data": "synthetic (seeded; signs Bernoulli(0.5), scales lognormal(-3,0.5) fp16, x N(0,1) bf16)",
            "config": {"workload": f"{w.key}: {w.title}", "layers": len(shapes), "M": M,
                       "l2": ("L2 flushed (256 MB write) before every step; steps timed alone" if args.flush_l2 else
                              "inputs larger than L2 (stack streams from HBM every step)"
                              if prefill_main or step_bytes > 126e6 else "stack fits in L2 (effective GB/s, warm)"),
                       "parallelism": f"replicas x{world}"},
            "tokens_per_s": round(world * M * args.steps / (total_ms * 1e-3), 1),
            "roofline": roof, "gpu_launches": res["launches"], "clocks": res["clocks"], "e2e": e2e}
    if not prefill_main:
        line["config"]["bytes_per_step"] = step_bytes

    if args.prefill and world == 1 and not prefill_main:
        line["prefill"] = run_prefill(args.prefill, args.prefill_steps, dev, pk, args.cpu_seconds)

    if args.configs and world == 1:
        line["configs"] = run_configs(args.configs, args.config_steps, dev, pk)

    if args.backward and world == 1:
        line["backward"] = run_backward(args.backward, args.backward_steps, 3, dev, args.cpu_seconds > 0, pk)

    if args.init and world == 1:
        line["init"] = run_init(args.init, args.init_steps, args.init_warmup, dev, args.cpu_seconds > 0,
                                args.init_layers)

    if rank == 0 and args.cpu_seconds > 0:
        cs = oracle_sample(w, M, args.cpu_seconds)
        cv = (cs["flops"] / cs["seconds"] / 1e12) if prefill_main else (cs["bytes"] / cs["seconds"] / 1e9)
        line["cpu_baseline"] = {"value": round(cv, 7), "unit": unit,
                                "cores": 1, "kind": "oracle",
                                "sample": f"first {cs['layers']} layers of the stack, {cs['rows']} of M={M} rows, "
                                          f"{cs['seconds']:.1f} s single-threaded float64 C"}
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line))


def e2e_of(res: dict, dist, world: int, work: float, prefill: bool, how: str):
    """End-to-end object (host buffers, copies inside the timed region) from run_gpu's e2e timings."""
    if not res["e2e"]:
        return None
    e_ms = max_over_ranks(res["e2e"]["ms"], dist)
    e_ser = max_over_ranks(res["e2e"]["serial_ms"], dist)
    scale, unit = (1e12, "TFLOP/s") if prefill else (1e9, "GB/s")
    return {"value": round(world * work / (e_ms * 1e-3) / scale, 2), "unit": unit,
            "h2d_bytes_per_step": res["e2e"]["h2d"], "d2h_bytes_per_step": res["e2e"]["d2h"],
            "ms_per_step": round(e_ms, 4),
            "how": how + ", steps pipelined: two device buffer sets, copies in and out on their own streams "
                         "overlap the previous/next step's compute",
            "serial": {"value": round(world * work / (e_ser * 1e-3) / scale, 2), "ms_per_step": round(e_ser, 4),
                       "how": "copy in, compute, copy out, one stream, no overlap"}}


def run_prefill(wkey: str, steps: int, dev, pk: dict, cpu_seconds: float):
    """The tensor-core (prefill) stack: throughput, roofline of the dominant GEMM, end to end on one block, and
    the oracle on a bounded sample."""
    pw = synth.WORKLOADS[wkey]
    pM = pw.Ms[0]
    pres = run_gpu(pw, pM, steps, 3, None, dev, want_e2e=False)
    pflops = sum(layer_flops(s, pM) for s in pres["shapes"])
    pms = pres["total_ms"] / steps
    tf = pflops / (pms * 1e-3) / 1e12
    out = {"workload": f"{pw.key}: {pw.title}", "M": pM, "layers": len(pres["shapes"]),
           "value": round(tf, 2), "unit": "TFLOP/s", "higher_is_better": True, "ms_per_step": round(pms, 3),
           "tokens_per_s": round(pM / (pms * 1e-3), 1), "steps": steps, "gpu_launches": pres["launches"],
           "l2": "inputs larger than L2 (every layer's x and weights are read from HBM)",
           "roofline": roofline_of(pres, pres["shapes"], pM, True, pk, pw.key),
           "step_traffic": prefill_traffic(pw.key), "clocks": pres["clocks"]}
    # end to end on the first block (its 7 layers): the full stack's host inputs and outputs (about 25 GB per
    # step) would be pinned twice over for the pipelined run
    bres = run_gpu(pw, pM, max(3, min(steps, 5)), 3, None, dev, want_e2e=True, nblocks=1)
    bflops = sum(layer_flops(s, pM) for s in bres["shapes"])
    out["e2e"] = e2e_of(bres, None, 1, bflops, True,
                        f"first block ({len(bres['shapes'])} layers) through lb_stack_forward from pinned host x "
                        f"[{pM} rows] to pinned host y")
    if cpu_seconds > 0:
        cs = oracle_sample(pw, pM, cpu_seconds)
        out["cpu_baseline"] = {"value": round(cs["flops"] / cs["seconds"] / 1e12, 9), "unit": "TFLOP/s",
                               "cores": 1, "kind": "oracle",
                               "sample": f"first {cs['layers']} layers of the stack, {cs['rows']} of M={pM} rows, "
                                         f"{cs['seconds']:.1f} s single-threaded float64 C"}
    return out


def run_configs(spec: str, steps: int, dev, pk: dict):
    """Decode throughput of the other workloads: one object per workload:M[:flushed] of `spec`."""
    out = []
    for item in [t for t in spec.split(",") if t]:
        parts = item.split(":")
        w = synth.WORKLOADS[parts[0]]
        M = int(parts[1]) if len(parts) > 1 else w.Ms[0]
        flushed = len(parts) > 2 and parts[2] == "flushed"
        res = run_gpu(w, M, steps, 5, None, dev, want_e2e=not flushed, flush_l2=flushed)
        shapes = res["shapes"]
        sb = sum(sum(layer_bytes(s, M)) for s in shapes)
        ms = res["total_ms"] / steps
        out.append({"workload": f"{w.key}: {w.title}", "M": M, "layers": len(shapes),
                    "e2e": e2e_of(res, None, 1, sb, False, "lb_stack_forward from pinned host x to pinned host y"),
                    "l2": ("L2 flushed (256 MB write) before every step; steps timed alone" if flushed else
                           "inputs larger than L2" if sb > 126e6 else "stack fits in L2 (effective GB/s, warm)"),
                    "value": round(sb / (ms * 1e-3) / 1e9, 2), "unit": "GB/s", "higher_is_better": True,
                    "ms_per_step": round(ms, 5), "tokens_per_s": round(M / (ms * 1e-3), 1),
                    "bytes_per_step": sb, "steps": steps, "gpu_launches": res["launches"],
                    "roofline": roofline_of(res, shapes, M, False, pk, w.key), "clocks": res["clocks"]})
    return out


def subspace_width(s: synth.LayerShape) -> int:
    """Columns of the subspace the initialisation iterates (include/littlebit_init.h)."""
    return min(min(s.N, s.K), max(64, -(-2 * s.r // 64) * 64))


def run_init(wkey: str, steps: int, warmup: int, dev, with_cpu: bool, only: str = ""):
    """Dual-SVID + residual initialisation of every layer of one block of a workload, from synthetic dense W.

    One step = both paths of all layers of the block (lb_dual_svid_init, binary64, INIT_ITERS iterations).  The
    dominant kernel is the binary64 GEMM of the subspace iteration; its launches are timed with the library's
    event hook on the largest layer.
    """
    import torch
    from sub_bit_weight_b200 import lib
    w = synth.WORKLOADS[wkey]
    shapes = [s for s in w.block if not only or s.name in only.split(",")]
    Ws = {}
    for s in shapes:        # one synthetic W per distinct shape (the work per layer does not depend on the values)
        if (s.N, s.K) not in Ws:
            Ws[(s.N, s.K)] = torch.from_numpy(synth.dense_weight(w.seed, s.N, s.K)).to(dev)
    ws = torch.empty(max(lib.lb_dual_svid_workspace_bytes(s.N, s.K, s.r) for s in shapes), dtype=torch.uint8,
                     device=dev)

    def block():
        for s in shapes:
            lib.lb_dual_svid_init(Ws[(s.N, s.K)], s.r, 2, INIT_ITERS, workspace=ws)

    for _ in range(warmup):
        block()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.nvtx.range_push("init_timed")
        e0.record()
        for _ in range(steps):
            block()
        e1.record()
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    ms_block = e0.elapsed_time(e1) / steps
    # the dominant kernel: the two products of the first subspace iteration of the largest layer
    big = max(shapes, key=lambda s: s.N * s.K * subspace_width(s))
    Lb = subspace_width(big)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
    for e in ev:             # torch creates the CUDA event on first record
        e.record()
    torch.cuda.synchronize()
    times = []
    for _ in range(3):
        lib.lb_profile_events(ev)
        lib.lb_dual_svid_init(Ws[(big.N, big.K)], big.r, 2, INIT_ITERS, workspace=ws)
        lib.lb_profile_events([])
        times += [ev[0].elapsed_time(ev[1]), ev[1].elapsed_time(ev[2])]
    gemm_ms = statistics.median(times)
    gemm_flops = 2.0 * big.N * big.K * Lb
    ach = gemm_flops / (gemm_ms * 1e-3) / 1e12
    # iteration products per layer and path: iters x 2 + the Rayleigh-Ritz product, each 2 N K L
    it_flops = sum(2 * (2 * INIT_ITERS + 1) * 2.0 * s.N * s.K * subspace_width(s) for s in shapes)
    out = {"workload": f"{w.key} first block: " + ", ".join(f"{s.name} {s.N}x{s.K} r={s.r}" for s in shapes)
                       + f"; dense W synthetic (power-law spectrum s_i ~ 1/i, bf16 values); two paths, "
                         f"{INIT_ITERS} subspace iterations, binary64",
           "value": round(len(shapes) / (ms_block * 1e-3), 3), "unit": "layers/s", "higher_is_better": True,
           "ms_per_block": round(ms_block, 2), "steps": steps, "warmup": warmup,
           "iteration_gemm_tflops": round(it_flops / (ms_block * 1e-3) / 1e12, 2),
           "roofline": {"bound": "alu", "kernel": f"dgemm_kernel (W^T (W Q) products, {big.name} {big.N}x{big.K}, "
                                                  f"L={Lb})",
                        "achieved": round(ach, 2), "peak": round(FP64_PEAK_TFLOPS, 1), "unit": "TFLOP/s",
                        "frac": round(ach / FP64_PEAK_TFLOPS, 4),
                        "peak_src": "derived: 148 SMs x 64 FP64 FMA/clk x 2 x 1965 MHz (binary64 CUDA-core rate)",
                        "flops_per_launch": gemm_flops, "ms_per_launch": round(gemm_ms, 4), "traffic": None},
           "clocks": clk.summary()}
    if with_cpu:
        from oracle import dual_svid as ods
        s = shapes[0]
        W = Ws[(s.N, s.K)].cpu().numpy().astype(np.float64)
        t = time.perf_counter()
        ods.littlebit_init(W, s.r, 2)
        dt = time.perf_counter() - t
        try:
            from threadpoolctl import threadpool_info
            cores = max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
        except Exception:
            cores = os.cpu_count()
        out["cpu_baseline"] = {"value": round(1.0 / dt, 4), "unit": "layers/s", "cores": cores, "kind": "oracle",
                               "sample": f"one {s.name} layer {s.N}x{s.K} r={s.r}, two paths, numpy/LAPACK "
                                         f"float64 ({dt:.1f} s)"}

    # LittleBit-2: the same block with the Joint-ITQ latent rotation before the binarisation (lb_littlebit2_init)
    ws2 = torch.empty(max(lib.lb_littlebit2_workspace_bytes(s.N, s.K, s.r) for s in shapes), dtype=torch.uint8,
                      device=dev)
    last = []

    def block2():
        last[:] = [lib.lb_littlebit2_init(Ws[(s.N, s.K)], s.r, 2, INIT_ITERS, ITQ_ITERS, workspace=ws2)
                   for s in shapes]

    for _ in range(warmup):
        block2()
    torch.cuda.synchronize()
    with ClockSampler(torch.cuda.current_device()) as clk2:
        torch.cuda.nvtx.range_push("littlebit2_timed")
        e0.record()
        for _ in range(steps):
            block2()
        e1.record()
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    ms2 = e0.elapsed_time(e1) / steps
    loss = np.array([r_.itq_loss.cpu().numpy() for r_ in last])       # [layer, path, ITQ_ITERS + 1]
    lb2 = {"value": round(len(shapes) / (ms2 * 1e-3), 3), "unit": "layers/s", "higher_is_better": True,
           "ms_per_block": round(ms2, 2), "itq_iters": ITQ_ITERS,
           "itq_ms_per_layer": round((ms2 - ms_block) / len(shapes), 2),
           "itq_loss_mean": {"start": round(float(loss[:, :, 0].mean()), 4),
                             "end": round(float(loss[:, :, -1].mean()), 4)},
           "clocks": clk2.summary()}
    if with_cpu:
        from oracle import littlebit2 as olb2
        s = shapes[0]
        W = Ws[(s.N, s.K)].cpu().numpy().astype(np.float64)
        t = time.perf_counter()
        olb2.littlebit2_init(W, s.r, 2, ITQ_ITERS)
        dt = time.perf_counter() - t
        lb2["cpu_baseline"] = {"value": round(1.0 / dt, 4), "unit": "layers/s", "cores": out["cpu_baseline"]["cores"],
                               "kind": "oracle", "sample": f"one {s.name} layer {s.N}x{s.K} r={s.r}, two paths, "
                                                           f"{ITQ_ITERS} ITQ alternations, numpy/LAPACK float64 "
                                                           f"({dt:.1f} s)"}
    out["littlebit2"] = lb2
    return out


def backward_stage_flops(s: synth.LayerShape, M: int, npaths: int = 2):
    """Algorithmic FLOPs of the backward stages of one layer (2 FLOPs per multiply-add, no padding)."""
    R = npaths * s.r
    return {"z = (x.g) V_s, (dy.h) U_s": 2.0 * M * (s.K + s.N) * R, "dx": 2.0 * M * R * s.K,
            "dy^T zl, x^T dz": 2.0 * M * (s.N + s.K) * R}


def run_backward(wkey: str, steps: int, warmup: int, dev, with_cpu: bool, pk):
    """QAT backward pass of every layer of one block of a workload (lb_layer_backward), M rows of the workload.

    One step = the backward of all layers of the block.  Inputs: latent factors N(0, 0.02) (their signs are the
    layer's), the workload's scales and activations, dy ~ N(0, 1) * 1e-4.  The dominant stage is timed with the
    library's event hook on the largest layer.
    """
    import torch
    from sub_bit_weight_b200 import lib
    w = synth.WORKLOADS[wkey]
    shapes = list(w.block)
    M = w.Ms[0]
    rng = np.random.default_rng(w.seed + 77)
    objs = {}
    for s in shapes:
        if (s.N, s.K) in objs:
            continue
        U = [torch.from_numpy(rng.normal(0, 0.02, (s.N, s.r)).astype(np.float32)).to(dev) for _ in range(2)]
        V = [torch.from_numpy(rng.normal(0, 0.02, (s.K, s.r)).astype(np.float32)).to(dev) for _ in range(2)]
        sc = {k: [torch.from_numpy(synth.scale_vector(w.seed, 0, p, k, n).view(np.int16)).to(dev) for p in range(2)]
              for k, n in (("h", s.N), ("g", s.K), ("l", s.r))}
        B = lib.lb_backward_create(s.N, s.K, s.r, [lib.lb_pack_signs(u) for u in U], [lib.lb_pack_signs(v) for v in V],
                                   sc["h"], sc["g"], sc["l"])
        x = torch.from_numpy(synth.activations(w.seed, 0, M, s.K).view(np.int16)).to(dev).view(torch.bfloat16)
        dy = torch.from_numpy((rng.standard_normal((M, s.N)) * 1e-4).astype(np.float32)).to(dev)
        objs[(s.N, s.K)] = (B, x, dy, U, V, sc)

    def block():
        for s in shapes:
            B, x, dy, U, V, _ = objs[(s.N, s.K)]
            lib.lb_layer_backward(B, x, dy, U, V)

    for _ in range(warmup):
        block()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(torch.cuda.current_device()) as clk:
        torch.cuda.nvtx.range_push("backward_timed")
        e0.record()
        for _ in range(steps):
            block()
        e1.record()
        torch.cuda.synchronize()
        torch.cuda.nvtx.range_pop()
    ms_block = e0.elapsed_time(e1) / steps
    flops = sum(sum(backward_stage_flops(s, M).values()) for s in shapes)
    tf = flops / (ms_block * 1e-3) / 1e12
    # stages of the largest layer, timed with the event hook (one event at every stage boundary)
    big = max(shapes, key=lambda s: s.N * s.K)
    B, x, dy, U, V, _ = objs[(big.N, big.K)]
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(9)]
    for e in ev:
        e.record()
    torch.cuda.synchronize()
    # events 2 and 3 mark the same point (z and dzl run in one launch), and so do 6 and 7 (dy^T zl and x^T dz);
    # after event 4 dx runs on the caller's stream (4 -> 5) beside the two dense products (4 -> 6) and the factor
    # gradients (7 -> 8) on a second stream
    spans = {"dy scaling": (0, 1), "z = (x.g) V_s, (dy.h) U_s": (1, 2), "dl, dz, zl": (3, 4), "dx": (4, 5),
             "dy^T zl, x^T dz": (4, 6), "dh, dg, dU, dV": (7, 8)}
    stage = {n: 0.0 for n in spans}
    reps = 5
    for _ in range(reps):
        lib.lb_profile_events(ev)
        lib.lb_layer_backward(B, x, dy, U, V)
        lib.lb_profile_events([])
        torch.cuda.synchronize()
        for n, (i, j) in spans.items():
            stage[n] += ev[i].elapsed_time(ev[j]) / reps
    sf = backward_stage_flops(big, M)
    dom = max(sf, key=lambda n: stage[n])
    ach = sf[dom] / (stage[dom] * 1e-3) / 1e12
    kern = {"z = (x.g) V_s, (dy.h) U_s": "prefill_kernel<0> (latent contractions of the forward and transposed "
                                         "helpers in one launch, k-split units)",
            "dx": "prefill_kernel<1> (output contraction of the transposed helper)",
            "dy^T zl, x^T dz": "gemm_at_b_kernel (tcgen05 fp16 GEMM, both operands MN-major, both products in one "
                               "launch)"}[dom]
    out = {"workload": f"{w.key} first block: " + ", ".join(f"{s.name} {s.N}x{s.K} r={s.r}" for s in shapes)
                       + f"; M = {M}, two paths; latent factors N(0, 0.02), dy N(0, 1) x 1e-4",
           "value": round(tf, 2), "unit": "TFLOP/s", "higher_is_better": True, "ms_per_block": round(ms_block, 3),
           "steps": steps, "warmup": warmup, "flops_per_block": flops,
           "stages_ms_largest_layer": {n: round(v, 4) for n, v in stage.items()},
           "roofline": {"bound": "tensor", "kernel": f"{dom}: {kern}, {big.name} {big.N}x{big.K}",
                        "achieved": round(ach, 1), "peak": pk["bf16_tflops_sustained"], "unit": "TFLOP/s",
                        "frac": round(ach / pk["bf16_tflops_sustained"], 4),
                        "peak_src": pk["src"] + " bf16 sustained (fp16 has the same dense rate)", "traffic": None},
           "clocks": clk.summary()}
    if with_cpu:
        from oracle import qat_backward as qb
        s = shapes[0]
        Bq, x, dy, U, V, sc = objs[(s.N, s.K)]
        f16 = lambda t: t.cpu().numpy().view(np.float16).astype(np.float64)
        xn = synth.bf16_bits_to_f32(x.view(torch.int16).cpu().numpy().view(np.uint16))
        t0 = time.perf_counter()
        qb.backward(xn, dy.cpu().numpy(), [u.cpu().numpy() for u in U], [v.cpu().numpy() for v in V],
                    [f16(v) for v in sc["h"]], [f16(v) for v in sc["g"]], [f16(v) for v in sc["l"]])
        dt = time.perf_counter() - t0
        try:
            from threadpoolctl import threadpool_info
            cores = max((i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"), default=1)
        except Exception:
            cores = os.cpu_count()
        of = sum(backward_stage_flops(s, M).values())
        out["cpu_baseline"] = {"value": round(of / dt / 1e12, 5), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                               "sample": f"one {s.name} layer {s.N}x{s.K} r={s.r}, M = {M}, numpy float64 ({dt:.1f} s)"}
    for v in objs.values():
        v[0].close()
    return out


def reference_arm(args, w, M, world, rank, pk):
    """The CPU oracle timed as it stands, on the same workload/metric (rank 0 only)."""
    if rank != 0:
        return
    # each step a bounded sample of the workload: at most --cpu-seconds of oracle time, the whole run a few minutes
    per_step = max(0.2, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, M, per_step / 4, max_layers=1)
    t_work = t_sec = 0.0
    layers = 0
    prefill = bool(w.pool_rows)
    for _ in range(args.steps):
        cs = oracle_sample(w, M, per_step)
        t_work += cs["flops"] if prefill else cs["bytes"]
        t_sec += cs["seconds"]
        layers += cs["layers"]
    v = t_work / t_sec / (1e12 if prefill else 1e9)
    unit = "TFLOP/s" if prefill else "GB/s"
    line = {"metric": METRIC, "value": round(v, 7), "unit": unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t_sec / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "impl": "reference",
            "config": {"workload": f"{w.key}: {w.title}", "M": M},
            "cpu_baseline": {"value": round(v, 7), "unit": unit, "cores": 1, "kind": "oracle",
                             "sample": f"{layers} layers over {args.steps} steps (first layers of the stack), "
                                       f"single-threaded float64 C"},
            "e2e": {"value": round(v, 7), "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


if __name__ == "__main__":
    main()
