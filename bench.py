"""Benchmark of the NVFP4 linear-layer hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl nvfp4|reference]
                    [--workload swiglu_block|quant_dense|quant_dense_fused|quant_masked|quant_silu|grouped_moe|
                                grouped_swiglu|lowrank|svdquant_linear|pr1_linear]
                    [--rank-lr R] [--swiglu-path fused|unfused] [--no-pdl]

Default workload: the dense NVFP4 SwiGLU shared-expert block, M = 8192 tokens, hidden
5120, intermediate 8192.  One step is the whole hot path over one batch:
    global amax of x (dynamic activation scale; also yields the gate/up alpha) and the
    quantization of x [8192, 5120] in one launch
    -> gate/up GEMM [8192 x 5120] @ [16384 x 5120]^T whose epilogue forms
       h = bf16(silu(gate) * up) and quantizes it with the calibrated static scale of h
       (--swiglu-path unfused: the pages' sequence of separate kernels -- amax, quantize,
       the GEMM writing bf16 [gate | up], the SiLU-and-mul quantizer)
    -> down GEMM [8192 x 8192] @ [5120 x 8192]^T  (bf16 out)
Weights are quantized once before timing (offline weight quantization), and the static
activation scale of h is calibrated once, as a deployed layer would.

Timing: the step is captured into a CUDA graph with event nodes only at its start and
end (its kernels chained by programmatic dependent launch unless --no-pdl), and into a
second graph with an event node around every kernel.  W warm-up replays, then K timed
replays of each graph, alternating (step graph, kernel graph) so both see the same clocks,
bracketed by a barrier and a device synchronize.  Before every
replay L2 is flushed outside the events (a 512 MB write, then a 256 MB read that leaves
no dirty line of the flush to be written back inside the timing).  ms_per_step and the
value come from the step graph; per-kernel times (parts, roofline) from the kernel
graph.  The value is whole-job throughput (sum over ranks of the work / the max over
ranks of the device time).  With N > 1 every rank runs its own independent batch (data
parallel, no collective on the data path): weak scaling.

On one GPU the default run then times every other configuration the same way (the PR1
linear, the quantize sweep -- dense, masked, SiLU-and-mul --, the masked grouped GEMM, the
low-rank GEMM at r = 32, 64, 128), each reported under ``configs`` with its value, its
dominant kernel's roofline, its parts and an oracle sample; and the headline's step graph
is replayed back to back for at least one second (``sustained``: the power-capped regime,
with its own clock record).  --no-configs / --no-sustained skip them.

``--impl reference`` times the CPU oracle (the plain C reference implementation) on a
bounded sample of the same workload on this machine's host cores.
"""
import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import nvfp4_synth as S  # noqa: E402

METRIC = "NVFP4 GEMM TFLOPS (% of FP4 peak); quantize HBM GB/s (% of HBM peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
FP4_OVER_BF16 = 4.0          # nominal dense ratio 9 PFLOP/s / 2.25 PFLOP/s
L2_FLUSH_BYTES = 512 << 20      # written before every step (L2 is 126 MB) ...
L2_CLEAN_BYTES = 256 << 20      # ... then read, so the flush's dirty lines are written back outside the timing
L2_NOTE = ("flushed before every step outside the timed events: 512 MB written, then 256 MB read so that "
           "no dirty line of the flush is written back inside the timing")


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def file_sha(path):
    with open(path, "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


# The CUDA kernel behind each launch name that can be a workload's dominant launch (the key of
# its DRAM traffic in profiles/traffic.json).
KERNEL_OF_LAUNCH = {
    "quantize": "quantize_kernel", "quantize_masked": "persistent_quantize_kernel",
    "silu_mul_quantize": "persistent_quantize_kernel", "global_scale_quantize": "global_scale_quantize_kernel",
    "global_scale_quantize_x": "global_scale_quantize_kernel",
    "quantize_smooth_lora_down": "svdquant_input_kernel",
}


def recorded_traffic(kernel, workload):
    """DRAM bytes per launch from a committed ncu summary, if the kernel source is unchanged."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(f"{kernel}@{workload}")
    if not e:
        return None
    src = os.path.join(ROOT, e["source"])
    if not os.path.exists(src) or file_sha(src) != e["source_sha"]:
        return None
    return e["bytes_per_launch"]


# ---------------------------------------------------------------------------------------
# distributed plumbing
# ---------------------------------------------------------------------------------------

def dist_setup(n_gpus):
    import torch
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


def _reduce(world, v, op, device):
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=op)
    return t.item()


def max_over_ranks(world, v, device="cuda"):
    import torch.distributed as dist
    return _reduce(world, v, dist.ReduceOp.MAX if world > 1 else None, device)


def sum_over_ranks(world, v, device="cuda"):
    import torch.distributed as dist
    return _reduce(world, v, dist.ReduceOp.SUM if world > 1 else None, device)


def aggregate(world, work_local, ms_local, device="cuda"):
    """Whole-job throughput of a data-parallel run: (sum over ranks of the work) / (max over
    ranks of the device time).  Returns (work of all ranks, max time in ms)."""
    return sum_over_ranks(world, work_local, device), max_over_ranks(world, ms_local, device)


# ---------------------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    _count = 0

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None
        ClockSampler._count += 1          # one file per sampler: a process may run several
        self.path = os.path.join("/tmp", f"nvfp4_clocks_{os.getpid()}_{ClockSampler._count}.csv")

    def __enter__(self):
        try:
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                                          "-i", str(self.gpu), "-lms", "20"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.1)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self, busy_only=True):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            p = [x.strip() for x in line.split(",")]
            if len(p) < 9:
                continue
            try:
                rows.append((float(p[1]), float(p[2]), float(p[3]) if p[3] not in ("[N/A]", "N/A") else 0.0, p[4:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] if busy_only else rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3][1:]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": pmax}


# ---------------------------------------------------------------------------------------
# workloads (GPU)
# ---------------------------------------------------------------------------------------

def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def quantize_weight(nv, w):
    """Offline weight quantization with the library: global scale, then block quantize."""
    amax, gsf, _ = nv.nvfp4_global_scale(w)
    q, sf = nv.nvfp4_quantize(w, gsf)
    return q, sf, amax


class Workload:
    name = ""
    unit = "TFLOP/s"
    dominant = ""

    def launches(self):
        """List of (kernel name, callable) making up one step on the current stream."""
        raise NotImplementedError

    def work(self):
        """Algorithmic work per step in the metric's unit base (FLOP or bytes)."""
        raise NotImplementedError


class SwigluBlock(Workload):
    """Dense SwiGLU block.  fused=True: amax(x) and quantize(x) in one launch, the gate/up
    GEMM whose epilogue emits SiLU(g)*u as NVFP4, the down GEMM.  fused=False: the pages'
    sequence of separate kernels -- amax(x), quantize(x), the gate/up GEMM writing bf16
    [g | u], the SiLU-and-mul quantizer, the down GEMM."""
    name = "swiglu_block"
    unit = "TFLOP/s"

    def __init__(self, nv, seed=0, fused=True):
        import torch
        self.nv = nv
        self.fused = fused
        self.dominant = "gemm_gate_up_silu_quantize" if fused else "gemm_gate_up"
        self.M, self.H, self.I = 8192, 5120, 8192
        d = S.swiglu_block(self.M, self.H, self.I, seed)
        self.x_host = d["x"]
        self.x = to_dev_bf16(d["x"])
        self.wgu_q, self.wgu_sf, self.amax_wgu = quantize_weight(nv, to_dev_bf16(d["w_gate_up"]))
        self.wd_q, self.wd_sf, self.amax_wd = quantize_weight(nv, to_dev_bf16(d["w_down"]))
        dev = self.x.device
        self.amax_x = torch.empty(1, dtype=torch.float32, device=dev)
        self.gsf_x = torch.empty(1, dtype=torch.float32, device=dev)
        self.alpha1 = torch.empty(1, dtype=torch.float32, device=dev)
        self.xq = torch.empty((self.M, self.H // 2), dtype=torch.uint8, device=dev)
        self.xsf = torch.empty(nv.nvfp4_scale_bytes(self.M, self.H), dtype=torch.uint8, device=dev)
        self.gu = torch.empty((self.M, 2 * self.I), dtype=torch.bfloat16, device=dev)
        self.hq = torch.empty((1, self.M, self.I // 2), dtype=torch.uint8, device=dev)
        self.hsf = torch.empty((1, nv.nvfp4_scale_bytes(self.M, self.I)), dtype=torch.uint8, device=dev)
        self.y = torch.empty((self.M, self.H), dtype=torch.bfloat16, device=dev)
        # the gate and up weights are the two row halves of the one quantized [2I, H] tensor
        half = nv.nvfp4_scale_bytes(self.I, self.H)
        self.wg_q, self.wu_q = self.wgu_q[:self.I], self.wgu_q[self.I:]
        self.wg_sf, self.wu_sf = self.wgu_sf[:half], self.wgu_sf[half:]
        # calibration pass (offline, unfused): static scale of h = silu(gate) * up and the
        # down-projection alpha
        self._unfused_launches()[0][1]()
        self._unfused_launches()[1][1]()
        self._unfused_launches()[2][1]()
        amax_h, self.gsf_h = nv.nvfp4_global_scale_batched(self.gu.view(1, self.M, 2 * self.I), None, silu_mul=True)
        if fused:
            del self.gu
        a_h = np.float32(amax_h.item())
        a_w = np.float32(self.amax_wd.item())
        self.alpha2 = torch.tensor([np.float32(a_h * a_w) / np.float32(7225344.0)], dtype=torch.float32, device=dev)
        torch.cuda.synchronize()

    def launches(self):
        if not self.fused:
            return self._unfused_launches()
        nv = self
        lib = self.nv
        return [
            ("global_scale_quantize_x", lambda: lib.nvfp4_global_scale_quantize(
                nv.x, nv.amax_wgu, nv.amax_x, nv.gsf_x, nv.alpha1, nv.xq, nv.xsf)),
            ("gemm_gate_up_silu_quantize", lambda: lib.nvfp4_gemm_silu_mul_quantize(
                nv.xq, nv.wg_q, nv.wu_q, nv.xsf, nv.wg_sf, nv.wu_sf, nv.alpha1, nv.alpha1, nv.gsf_h,
                nv.hq.view(nv.M, nv.I // 2), nv.hsf.view(-1))),
            ("gemm_down", lambda: lib.nvfp4_gemm(nv.hq.view(nv.M, nv.I // 2), nv.wd_q, nv.hsf.view(-1), nv.wd_sf,
                                                 nv.alpha2, None, nv.y)),
        ]

    def _unfused_launches(self):
        nv = self
        lib = self.nv
        return [
            ("global_scale_x", lambda: lib.nvfp4_global_scale(nv.x, nv.amax_x, nv.gsf_x, nv.amax_wgu, nv.alpha1)),
            ("quantize_x", lambda: lib.nvfp4_quantize(nv.x, nv.gsf_x, nv.xq, nv.xsf)),
            ("gemm_gate_up", lambda: lib.nvfp4_gemm(nv.xq, nv.wgu_q, nv.xsf, nv.wgu_sf, nv.alpha1, None, nv.gu)),
            ("silu_mul_quantize", lambda: lib.nvfp4_silu_mul_quantize_batched(
                nv.gu.view(1, nv.M, 2 * nv.I), nv.gsf_h, None, nv.hq, nv.hsf)),
            ("gemm_down", lambda: lib.nvfp4_gemm(nv.hq.view(nv.M, nv.I // 2), nv.wd_q, nv.hsf.view(-1), nv.wd_sf,
                                                 nv.alpha2, None, nv.y)),
        ]

    def work(self):
        return 2.0 * self.M * self.H * (2 * self.I) + 2.0 * self.M * self.I * self.H

    def kernel_work(self):
        M, H, I = self.M, self.H, self.I
        names = {name for name, _ in self.launches()}
        return {k: v for k, v in {
            "global_scale_x": (2.0 * M * H, "GB/s"),
            "quantize_x": (2.5625 * M * H, "GB/s"),
            "global_scale_quantize_x": (2.5625 * M * H, "GB/s"),
            "gemm_gate_up": (2.0 * M * H * 2 * I, "TFLOP/s"),
            "gemm_gate_up_silu_quantize": (2.0 * M * H * 2 * I, "TFLOP/s"),
            "silu_mul_quantize": (4.5625 * M * I, "GB/s"),
            "gemm_down": (2.0 * M * I * H, "TFLOP/s"),
        }.items() if k in names}

    def e2e_io(self):
        """(host input, device input, device output) of the end-to-end measurement."""
        return self.x_host, self.x, self.y

    def config(self):
        return {"workload": "dense NVFP4 SwiGLU shared-expert block: tokens M=8192, hidden K=5120, "
                            "intermediate 8192; gate/up [8192x5120]@[16384x5120]^T, silu*mul requantize, "
                            "down [8192x8192]@[5120x8192]^T; x~N(0,1), W~N(0,0.02)",
                "tokens": self.M, "hidden": self.H, "intermediate": self.I,
                "path": ("amax and quantize of x in one launch, gate/up GEMM with the SiLU*mul NVFP4 quantizer "
                         "in its epilogue, down GEMM" if self.fused else
                         "amax, quantize, gate/up GEMM to bf16, SiLU*mul quantizer, down GEMM (separate kernels)"),
                "l2": L2_NOTE}


class QuantDense(Workload):
    name = "quant_dense"
    unit = "GB/s"
    dominant = "quantize"

    def __init__(self, nv, seed=0):
        import torch
        self.nv = nv
        self.m = self.k = 8192
        self.x_host = S.quant_dense(self.m, self.k, seed)["x"]
        self.x = to_dev_bf16(self.x_host)
        self.amax = torch.empty(1, dtype=torch.float32, device="cuda")
        self.gsf = torch.empty(1, dtype=torch.float32, device="cuda")
        self.q = torch.empty((self.m, self.k // 2), dtype=torch.uint8, device="cuda")
        self.sf = torch.empty(nv.nvfp4_scale_bytes(self.m, self.k), dtype=torch.uint8, device="cuda")

    def launches(self):
        lib, s = self.nv, self
        return [("global_scale", lambda: lib.nvfp4_global_scale(s.x, s.amax, s.gsf)),
                ("quantize", lambda: lib.nvfp4_quantize(s.x, s.gsf, s.q, s.sf))]

    def work(self):
        return 2.5625 * self.m * self.k

    def kernel_work(self):
        return {"global_scale": (2.0 * self.m * self.k, "GB/s"), "quantize": (2.5625 * self.m * self.k, "GB/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.q

    def config(self):
        return {"workload": "quantize bf16 [8192,8192] ~N(0,1) with 0.1% outliers x50 (amax + quantize)",
                "l2": L2_NOTE}


class QuantDenseFused(QuantDense):
    """The quant_dense workload through nvfp4_global_scale_quantize: amax and quantize in
    one launch."""
    name = "quant_dense_fused"
    dominant = "global_scale_quantize"

    def launches(self):
        lib, s = self.nv, self
        return [("global_scale_quantize", lambda: lib.nvfp4_global_scale_quantize(s.x, None, s.amax, s.gsf, None,
                                                                                   s.q, s.sf))]

    def kernel_work(self):
        return {"global_scale_quantize": (2.5625 * self.m * self.k, "GB/s")}

    def config(self):
        return {"workload": "quantize bf16 [8192,8192] ~N(0,1) with 0.1% outliers x50 (amax and quantize in one "
                            "launch)", "l2": L2_NOTE}


class QuantMasked(Workload):
    unit = "GB/s"
    dominant = "quantize_masked"

    def __init__(self, nv, silu, seed=0):
        import torch
        self.nv, self.silu = nv, silu
        self.name = "quant_silu" if silu else "quant_masked"
        self.dominant = "silu_mul_quantize" if silu else "quantize_masked"
        self.b, self.m, self.k = 8, 4096, 7168
        d = S.quant_silu(self.b, self.m, self.k, seed) if silu else S.quant_masked(self.b, self.m, self.k, seed)
        self.x_host = d["x"]
        self.x = to_dev_bf16(d["x"])
        self.mask_host = d["mask"]
        self.mask = torch.from_numpy(d["mask"]).cuda()
        _, self.gsf = nv.nvfp4_global_scale_batched(self.x, self.mask, silu_mul=silu)
        self.q = torch.empty((self.b, self.m, self.k // 2), dtype=torch.uint8, device="cuda")
        self.sf = torch.empty((self.b, nv.nvfp4_scale_bytes(self.m, self.k)), dtype=torch.uint8, device="cuda")
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        fn = lib.nvfp4_silu_mul_quantize_batched if self.silu else lib.nvfp4_quantize_masked_batched
        return [(self.dominant, lambda: fn(s.x, s.gsf, s.mask, s.q, s.sf))]

    def work(self):
        per_row = (4 * self.k + self.k // 2 + self.k // 16) if self.silu else (2 * self.k + self.k // 2 + self.k // 16)
        return float(per_row * int(self.mask_host.sum()))

    def kernel_work(self):
        return {self.dominant: (self.work(), "GB/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.q

    def config(self):
        w = "[8,4096,2*7168] silu(gate)*up fused" if self.silu else "[8,4096,7168]"
        return {"workload": f"masked batched quantize {w}, valid rows per item U[0,4096] (sum {int(self.mask_host.sum())})",
                "l2": L2_NOTE}


class GroupedMoE(Workload):
    name = "grouped_moe"
    unit = "TFLOP/s"
    dominant = "grouped_gemm"

    def __init__(self, nv, seed=0):
        import torch
        self.nv = nv
        self.E, self.mmax, self.k, self.n = 16, 2048, 5120, 8192
        d = S.grouped_moe(self.E, self.mmax, self.k, self.n, 512, seed)
        self.mask_host = d["mask"]
        self.mask = torch.from_numpy(d["mask"]).cuda()
        a = to_dev_bf16(d["a"])
        w = to_dev_bf16(d["w"])
        amax_a, ga = nv.nvfp4_global_scale_batched(a, self.mask)
        amax_w, gw = nv.nvfp4_global_scale_batched(w, None)
        self.aq, self.asf = nv.nvfp4_quantize_masked_batched(a, ga, self.mask)
        self.wq, self.wsf = nv.nvfp4_quantize_masked_batched(w, gw, None)
        al = (amax_a.cpu().numpy().astype(np.float32) * amax_w.cpu().numpy().astype(np.float32)) / np.float32(7225344.0)
        self.alpha = torch.from_numpy(al.astype(np.float32)).cuda()
        self.out = torch.empty((self.E, self.mmax, self.n), dtype=torch.bfloat16, device="cuda")
        self.a_host = d["a"]
        del a, w
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        return [("grouped_gemm", lambda: lib.nvfp4_grouped_gemm_masked(s.aq, s.wq, s.asf, s.wsf, s.mask, s.alpha,
                                                                        s.out))]

    def work(self):
        return 2.0 * int(self.mask_host.sum()) * self.n * self.k

    def kernel_work(self):
        return {"grouped_gemm": (self.work(), "TFLOP/s")}

    def e2e_io(self):
        return None

    def config(self):
        return {"workload": f"masked grouped NVFP4 GEMM E=16 Mmax=2048 K=5120 N=8192, valid rows "
                            f"min(Poisson(512),2048) (sum {int(self.mask_host.sum())})",
                "l2": L2_NOTE}


class GroupedSwiglu(Workload):
    """Routed-expert SwiGLU: masked quantize of every expert's tokens, the grouped gate/up
    GEMM whose epilogue emits SiLU(g)*u as NVFP4, the grouped down GEMM.  Activation scales
    (x and h, per expert) are static, calibrated once, as the masked quantizer's global
    scale input is."""
    name = "grouped_swiglu"
    unit = "TFLOP/s"
    dominant = "grouped_gemm_gate_up_silu_quantize"

    def __init__(self, nv, seed=0):
        import torch
        self.nv = nv
        self.E, self.mmax, self.H, self.I = 16, 2048, 5120, 8192
        d = S.grouped_swiglu(self.E, self.mmax, self.H, self.I, 512, seed)
        E, mmax, H, I = self.E, self.mmax, self.H, self.I
        self.mask_host = d["mask"]
        self.mask = torch.from_numpy(d["mask"]).cuda()
        self.x_host = d["x"]
        self.x = to_dev_bf16(d["x"])
        amax_x, self.gsf_x = nv.nvfp4_global_scale_batched(self.x, self.mask)      # calibration
        amaxes = {}
        for name in ("w_gate", "w_up", "w_down"):
            w = to_dev_bf16(d[name])
            amax, g = nv.nvfp4_global_scale_batched(w, None)
            q, sf = nv.nvfp4_quantize_masked_batched(w, g, None)
            setattr(self, name + "_q", q)
            setattr(self, name + "_sf", sf)
            amaxes[name] = amax.cpu().numpy().astype(np.float32)
            del w
        ax = amax_x.cpu().numpy().astype(np.float32)

        def alpha(a, b):
            return torch.from_numpy(((a * b) / np.float32(7225344.0)).astype(np.float32)).cuda()

        self.alpha_g = alpha(ax, amaxes["w_gate"])
        self.alpha_u = alpha(ax, amaxes["w_up"])
        self.xq = torch.empty((E, mmax, H // 2), dtype=torch.uint8, device="cuda")
        self.xsf = torch.empty((E, nv.nvfp4_scale_bytes(mmax, H)), dtype=torch.uint8, device="cuda")
        self.hq = torch.empty((E, mmax, I // 2), dtype=torch.uint8, device="cuda")
        self.hsf = torch.empty((E, nv.nvfp4_scale_bytes(mmax, I)), dtype=torch.uint8, device="cuda")
        self.y = torch.empty((E, mmax, H), dtype=torch.bfloat16, device="cuda")
        # calibration of the static h scales (offline, unfused): [g | u] in bf16, amax of silu(g)*u
        nv.nvfp4_quantize_masked_batched(self.x, self.gsf_x, self.mask, self.xq, self.xsf)
        g = nv.nvfp4_grouped_gemm_masked(self.xq, self.w_gate_q, self.xsf, self.w_gate_sf, self.mask, self.alpha_g)
        u = nv.nvfp4_grouped_gemm_masked(self.xq, self.w_up_q, self.xsf, self.w_up_sf, self.mask, self.alpha_u)
        gu = torch.cat([g, u], dim=-1)
        del g, u
        amax_h, self.gsf_h = nv.nvfp4_global_scale_batched(gu, self.mask, silu_mul=True)
        del gu
        self.alpha_d = alpha(amax_h.cpu().numpy().astype(np.float32), amaxes["w_down"])
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        return [
            ("quantize_x_masked", lambda: lib.nvfp4_quantize_masked_batched(s.x, s.gsf_x, s.mask, s.xq, s.xsf)),
            ("grouped_gemm_gate_up_silu_quantize", lambda: lib.nvfp4_grouped_gemm_silu_mul_quantize_masked(
                s.xq, s.w_gate_q, s.w_up_q, s.xsf, s.w_gate_sf, s.w_up_sf, s.mask, s.alpha_g, s.alpha_u, s.gsf_h,
                s.hq, s.hsf)),
            ("grouped_gemm_down", lambda: lib.nvfp4_grouped_gemm_masked(s.hq, s.w_down_q, s.hsf, s.w_down_sf, s.mask,
                                                                        s.alpha_d, s.y)),
        ]

    def work(self):
        return 6.0 * int(self.mask_host.sum()) * self.H * self.I

    def kernel_work(self):
        rows = int(self.mask_host.sum())
        return {"quantize_x_masked": (2.5625 * rows * self.H, "GB/s"),
                "grouped_gemm_gate_up_silu_quantize": (4.0 * rows * self.H * self.I, "TFLOP/s"),
                "grouped_gemm_down": (2.0 * rows * self.I * self.H, "TFLOP/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.y

    def config(self):
        return {"workload": f"routed-expert NVFP4 SwiGLU, E=16 experts, Mmax=2048 tokens each, valid rows "
                            f"min(Poisson(512),2048) (sum {int(self.mask_host.sum())}), hidden 5120, "
                            f"intermediate 8192; masked quantize, grouped gate/up GEMM with the SiLU*mul NVFP4 "
                            f"epilogue, grouped down GEMM; static per-expert activation scales",
                "experts": self.E, "mmax": self.mmax, "hidden": self.H, "intermediate": self.I,
                "l2": L2_NOTE}


class LowRank(Workload):
    name = "lowrank"
    unit = "TFLOP/s"
    dominant = "gemm_lowrank"

    def __init__(self, nv, r=64, seed=0):
        import torch
        self.nv, self.r = nv, r
        self.m, self.k, self.n = 4096, 3072, 3072
        d = S.lowrank(self.m, self.k, self.n, r, seed)
        x = to_dev_bf16(d["x"])
        amax_x, gsf_x, _ = nv.nvfp4_global_scale(x)
        self.xq, self.xsf = nv.nvfp4_quantize(x, gsf_x)
        self.wq, self.wsf, amax_w = quantize_weight(nv, to_dev_bf16(d["w"]))
        alpha = np.float32(np.float32(amax_x.item()) * np.float32(amax_w.item())) / np.float32(7225344.0)
        self.alpha = torch.tensor([alpha], dtype=torch.float32, device="cuda")
        self.d = to_dev_bf16(d["d"])
        self.l1 = to_dev_bf16(S.f32_to_bf16_bits(d["l1_f32"] / alpha))
        self.bias = to_dev_bf16(d["bias"])
        self.out = torch.empty((self.m, self.n), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        return [("gemm_lowrank", lambda: lib.nvfp4_gemm_lowrank_bias(s.xq, s.wq, s.xsf, s.wsf, s.alpha, s.d, s.l1,
                                                                      s.bias, s.out))]

    def work(self):
        return 2.0 * self.m * self.n * self.k + 2.0 * self.m * self.n * self.r

    def kernel_work(self):
        return {"gemm_lowrank": (self.work(), "TFLOP/s")}

    def e2e_io(self):
        return None

    def config(self):
        return {"workload": f"low-rank-corrected NVFP4 GEMM M=4096 K=3072 N=3072 r={self.r} + bias",
                "l2": L2_NOTE}


class SvdquantLinear(Workload):
    """The whole SVDQuant NVFP4 linear layer at the low-rank GEMM's sizes: smooth quantize of x
    and the LoRA-down product in one pass (nvfp4_quantize_smooth_lora_down), then the residual
    FP4 GEMM with the rank-r correction and bias.  The activation scale of x_hat is static
    (calibrated once)."""
    name = "svdquant_linear"
    unit = "TFLOP/s"
    dominant = "gemm_lowrank"

    def __init__(self, nv, r=64, seed=0):
        import torch
        self.nv, self.r = nv, r
        self.m, self.k, self.n = 4096, 3072, 3072
        d = S.svdquant_linear(self.m, self.k, self.n, r, seed)
        self.x_host = d["x"]
        self.x = to_dev_bf16(d["x"])
        self.pqs = to_dev_bf16(d["pqs"])
        self.w_down = to_dev_bf16(d["w_down"])
        # calibration (offline): amax of x_hat = bf16(x * pre_quant_scale)
        xh = S.f32_to_bf16_bits(S.bf16_bits_to_f32(d["x"]) * S.bf16_bits_to_f32(d["pqs"])[None, :])
        amax_x = np.float32(np.abs(S.bf16_bits_to_f32(xh)).max())
        self.gsf = torch.tensor([np.float32(2688.0) / amax_x], dtype=torch.float32, device="cuda")
        self.wq, self.wsf, amax_w = quantize_weight(nv, to_dev_bf16(d["w"]))
        alpha = np.float32(amax_x * np.float32(amax_w.item())) / np.float32(7225344.0)
        self.alpha = torch.tensor([alpha], dtype=torch.float32, device="cuda")
        self.l1 = to_dev_bf16(S.f32_to_bf16_bits(d["l1_f32"] / alpha))
        self.bias = to_dev_bf16(d["bias"])
        self.xq = torch.empty((self.m, self.k // 2), dtype=torch.uint8, device="cuda")
        self.xsf = torch.empty((nv.nvfp4_scale_bytes(self.m, self.k),), dtype=torch.uint8, device="cuda")
        self.dd = torch.empty((self.m, r), dtype=torch.bfloat16, device="cuda")
        self.out = torch.empty((self.m, self.n), dtype=torch.bfloat16, device="cuda")
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        return [("quantize_smooth_lora_down", lambda: lib.nvfp4_quantize_smooth_lora_down(
                    s.x, s.pqs, s.gsf, s.w_down, s.xq, s.xsf, s.dd)),
                ("gemm_lowrank", lambda: lib.nvfp4_gemm_lowrank_bias(s.xq, s.wq, s.xsf, s.wsf, s.alpha, s.dd, s.l1,
                                                                      s.bias, s.out))]

    def work(self):
        return 2.0 * self.m * self.n * self.k + 2.0 * self.m * self.n * self.r + 2.0 * self.m * self.k * self.r

    def kernel_work(self):
        m, n, k, r = self.m, self.n, self.k, self.r
        # input stage: HBM-bound (x read; codes, scales and d written)
        return {"quantize_smooth_lora_down": (2.0 * m * k + 0.5625 * m * k + 2.0 * m * r, "GB/s"),
                "gemm_lowrank": (2.0 * m * n * k + 2.0 * m * n * r, "TFLOP/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.out

    def config(self):
        return {"workload": f"SVDQuant NVFP4 linear layer M=4096 K=3072 N=3072 r={self.r} + bias: smooth quantize "
                            f"and LoRA-down in one pass over x, then the residual FP4 GEMM with the rank-r "
                            f"correction; x~N(0,1), pre_quant_scale~U[0.25,4], static x_hat scale",
                "l2": L2_NOTE}


class Bf16aLinear(Workload):
    """The bf16-activation NVFP4 linear (nvfp4_gemm_bf16a: the pages' f16a_nvfp4weight_scaled_mm
    in its compiled form) at the SwiGLU block's gate/up shape: x [8192, 5120] bf16, NVFP4
    weight [16384, 5120], bf16 out."""
    name = "bf16a_linear"
    unit = "TFLOP/s"
    dominant = "gemm"

    def __init__(self, nv, seed=0):
        import torch
        self.nv = nv
        self.M, self.K, self.N = 8192, 5120, 16384
        d = S.swiglu_block(self.M, self.K, self.N // 2, seed)
        self.x_host = d["x"]
        self.x = to_dev_bf16(d["x"])
        self.wq, self.wsf, self.amax_w = quantize_weight(nv, to_dev_bf16(d["w_gate_up"]))
        dev = self.x.device
        self.aq = torch.empty((self.M, self.K // 2), dtype=torch.uint8, device=dev)
        self.asf = torch.empty(nv.nvfp4_scale_bytes(self.M, self.K), dtype=torch.uint8, device=dev)
        self.scalars = torch.empty(3, dtype=torch.float32, device=dev)
        self.out = torch.empty((self.M, self.N), dtype=torch.bfloat16, device=dev)
        torch.cuda.synchronize()

    def launches(self):
        lib, s = self.nv, self
        # nvfp4_gemm_bf16a is these two launches; they are listed separately so that the
        # kernel pass times each
        return [("global_scale_quantize", lambda: lib.nvfp4_global_scale_quantize(
                    s.x, s.amax_w, s.scalars[0:1], s.scalars[1:2], s.scalars[2:3], s.aq, s.asf)),
                ("gemm", lambda: lib.nvfp4_gemm(s.aq, s.wq, s.asf, s.wsf, s.scalars[2:3], None, s.out))]

    def work(self):
        return 2.0 * self.M * self.N * self.K

    def kernel_work(self):
        return {"global_scale_quantize": (2.5625 * self.M * self.K, "GB/s"), "gemm": (self.work(), "TFLOP/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.out

    def config(self):
        return {"workload": "bf16-activation NVFP4 linear (dynamic activation scale and quantization, then the FP4 "
                            "GEMM) x [8192,5120] ~N(0,1), W [16384,5120] ~N(0,0.02), bf16 out",
                "l2": L2_NOTE}


class PR1Linear(Workload):
    name = "pr1_linear"
    unit = "TFLOP/s"
    dominant = "gemm"

    def __init__(self, nv, seed=0):
        import torch
        self.nv = nv
        d = S.pr1_linear(seed)
        self.x = to_dev_bf16(d["x"])
        self.wq, self.wsf, self.amax_w = quantize_weight(nv, to_dev_bf16(d["w"]))
        self.amax = torch.empty(1, dtype=torch.float32, device="cuda")
        self.gsf = torch.empty(1, dtype=torch.float32, device="cuda")
        self.alpha = torch.empty(1, dtype=torch.float32, device="cuda")
        self.xq = torch.empty((128, 128), dtype=torch.uint8, device="cuda")
        self.xsf = torch.empty(nv.nvfp4_scale_bytes(128, 256), dtype=torch.uint8, device="cuda")
        self.out = torch.empty((128, 256), dtype=torch.bfloat16, device="cuda")
        self.x_host = d["x"]

    def launches(self):
        lib, s = self.nv, self
        return [("global_scale_quantize", lambda: lib.nvfp4_global_scale_quantize(s.x, s.amax_w, s.amax, s.gsf, s.alpha,
                                                                                   s.xq, s.xsf)),
                ("gemm", lambda: lib.nvfp4_gemm(s.xq, s.wq, s.xsf, s.wsf, s.alpha, None, s.out))]

    def work(self):
        return 2.0 * 128 * 256 * 256

    def kernel_work(self):
        return {"gemm": (self.work(), "TFLOP/s")}

    def e2e_io(self):
        return self.x_host, self.x, self.out

    def config(self):
        return {"workload": "single NVFP4 linear x[128,256] W[256,256] (latency-bound): amax and quantize of x in "
                            "one launch, then the GEMM", "l2": L2_NOTE}


def workload_config(name, rank_lr, swiglu_path="fused"):
    """The `config` of a workload without a GPU: its sizes and its seeded masks only (the
    reference arm prints the same config as the CUDA arm)."""
    cls = {"swiglu_block": SwigluBlock, "quant_dense": QuantDense, "quant_dense_fused": QuantDenseFused,
           "quant_masked": QuantMasked, "quant_silu": QuantMasked, "grouped_moe": GroupedMoE,
           "grouped_swiglu": GroupedSwiglu, "lowrank": LowRank, "svdquant_linear": SvdquantLinear,
           "pr1_linear": PR1Linear, "bf16a_linear": Bf16aLinear}[name]
    w = cls.__new__(cls)
    w.fused = swiglu_path == "fused"
    w.M, w.H, w.I = 8192, 5120, 8192
    w.silu = name == "quant_silu"
    w.r = rank_lr
    w.E, w.mmax = 16, 2048
    if name in ("quant_masked", "quant_silu"):
        w.mask_host = S.masks_uniform(8, 4096, 0)
    elif name in ("grouped_moe", "grouped_swiglu"):
        w.mask_host = S.masks_poisson(16, 512, 2048, 0)
    return w.config()


def make_workload(name, nv, rank_lr, swiglu_path="fused"):
    if name == "swiglu_block":
        return SwigluBlock(nv, fused=swiglu_path == "fused")
    if name == "quant_dense":
        return QuantDense(nv)
    if name == "quant_dense_fused":
        return QuantDenseFused(nv)
    if name == "quant_masked":
        return QuantMasked(nv, False)
    if name == "quant_silu":
        return QuantMasked(nv, True)
    if name == "grouped_moe":
        return GroupedMoE(nv)
    if name == "grouped_swiglu":
        return GroupedSwiglu(nv)
    if name == "lowrank":
        return LowRank(nv, rank_lr)
    if name == "svdquant_linear":
        return SvdquantLinear(nv, rank_lr)
    if name == "pr1_linear":
        return PR1Linear(nv)
    if name == "bf16a_linear":
        return Bf16aLinear(nv)
    raise SystemExit(f"unknown workload {name}")


def scale(v, unit):
    return v / 1e12 if unit == "TFLOP/s" else v / 1e9


# ---------------------------------------------------------------------------------------
# CPU oracle timing (reference arm and cpu_baseline)
# ---------------------------------------------------------------------------------------

def host_cpu():
    """The host's CPU model and logical CPU count, reported beside the oracle's timing."""
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"cpu_model": model, "host_cpus": os.cpu_count()}


class OracleSample:
    """The CPU oracle on a bounded sample of a workload: ``setup()`` prepares (and
    quantizes, offline) the weights once; each ``step()`` runs the sample's hot path and
    returns its work in the metric's unit base and the seconds it took."""

    def __init__(self, workload, rows=None):
        import oracle as O
        self.O = O
        self.workload = workload
        self.threads = O.get_threads()
        self.unit = "GB/s" if workload.startswith("quant") else "TFLOP/s"
        w = workload
        if w == "swiglu_block":
            self.rows = rows or 48          # ~10 s of the oracle on 16 host threads
            d = S.swiglu_block(8192, 5120, 8192, 0)
            self.x = d["x"][:self.rows].copy()
            self.wgu, self.wd = d["w_gate_up"], d["w_down"]
            self.H, self.I = 5120, 8192
            self.sample = f"{self.rows} of 8192 token rows through the whole block (amax, quantize, gate/up GEMM, " \
                          f"SiLU-mul quantize, down GEMM)"
        elif w == "grouped_swiglu":
            self.rows = rows or 2
            d = S.grouped_swiglu(16, 2048, 5120, 8192, 512, 0, experts=1)
            self.x = d["x"][0, :self.rows].copy()
            self.wg, self.wu, self.wd = d["w_gate"][0], d["w_up"][0], d["w_down"][0]
            self.H, self.I = 5120, 8192
            self.sample = f"{self.rows} token rows of expert 0 through the routed-expert block (quantize, gate/up " \
                          f"GEMMs, SiLU-mul quantize, down GEMM)"
        elif w == "pr1_linear":
            self.rows = 128
            d = S.pr1_linear(0)
            self.x, self.w = d["x"], d["w"]
            self.sample = "the whole 128x256x256 linear (amax, quantize, GEMM)"
        elif w in ("quant_dense", "quant_dense_fused", "quant_masked", "quant_silu"):
            self.rows = rows or 256
            if w in ("quant_dense", "quant_dense_fused"):
                self.x = S.quant_dense(8192, 8192, 0)["x"][:self.rows].copy()
            else:
                k = 7168
                self.x = S.normal_bf16((1, self.rows, 2 * k if w == "quant_silu" else k), 1.0, 0, S.TID["x"])
            self.sample = f"{self.rows} valid rows"
        elif w == "svdquant_linear":
            self.rows = rows or 2
            d = S.svdquant_linear(4096, 3072, 3072, 64, 0)
            self.x = d["x"][:self.rows].copy()
            self.pqs, self.wd, self.w = d["pqs"], d["w_down"], d["w"]
            self.l1_f32, self.bias = d["l1_f32"], d["bias"]
            self.m, self.k, self.n = self.rows, 3072, 3072
            self.sample = f"{self.rows} token rows through the SVDQuant layer (smooth quantize, LoRA-down, residual " \
                          f"GEMM with the rank-64 correction and bias)"
        elif w in ("grouped_moe", "lowrank"):
            self.rows = rows or 2
            self.m, self.k, self.n = (self.rows, 5120, 8192) if w == "grouped_moe" else (self.rows, 3072, 3072)
            self.x = S.normal_bf16((self.m, self.k), 1.0, 0, S.TID["x"])
            self.w = S.normal_bf16((self.n, self.k), 0.02, 0, S.TID["w"])
            self.sample = f"{self.m} rows x N={self.n} x K={self.k}"
        elif w == "bf16a_linear":
            self.rows = rows or 64          # ~10 s of the oracle on 16 host threads
            d = S.swiglu_block(8192, 5120, 8192, 0)
            self.x = d["x"][:self.rows].copy()
            self.w = d["w_gate_up"]
            self.m, self.k, self.n = self.rows, 5120, 16384
            self.sample = f"{self.rows} of 8192 activation rows (global scale of the rows, quantize, GEMM against " \
                          f"the [16384, 5120] weight)"
        else:
            raise SystemExit(f"no oracle sample for {w}")
        self._setup()

    def _setup(self):
        O = self.O
        if self.workload == "swiglu_block":
            self.aw, gw = O.global_scale(self.wgu)
            self.qw, self.sfw = O.quantize(self.wgu, gw)
            self.ad, gd = O.global_scale(self.wd)
            self.qd, self.sfd = O.quantize(self.wd, gd)
        elif self.workload == "grouped_swiglu":
            self.ag, gg = O.global_scale(self.wg)
            self.qg, self.sfg = O.quantize(self.wg, gg)
            self.au, gu = O.global_scale(self.wu)
            self.qu, self.sfu = O.quantize(self.wu, gu)
            self.ad, gd = O.global_scale(self.wd)
            self.qd, self.sfd = O.quantize(self.wd, gd)
            self.ax, self.gx = O.global_scale(self.x)          # static activation scale (calibration)
        elif self.workload in ("pr1_linear", "grouped_moe", "lowrank", "svdquant_linear", "bf16a_linear"):
            self.aw, gw = O.global_scale(self.w)
            self.qw, self.sfw = O.quantize(self.w, gw)

    def step(self):
        O = self.O
        w = self.workload
        t0 = time.perf_counter()
        if w == "swiglu_block":
            rows, H, I = self.rows, self.H, self.I
            ax, gx = O.global_scale(self.x)
            qx, sfx = O.quantize(self.x, gx)
            al = O.alpha(float(ax), float(self.aw))
            half = O.scale_bytes(I, H)
            gu_bits = O.gemm_gate_up_bf16(qx, self.qw[:I], self.qw[I:], sfx, self.sfw[:half], self.sfw[half:],
                                          al, al, I, H, np.arange(rows)).reshape(1, rows, 2 * I)
            ah, gh = O.global_scale_batched(gu_bits, None, silu_mul=True)
            hq, hsf = O.silu_mul_quantize_batched(gu_bits, gh)
            O.gemm_ref(hq[0], self.qd, hsf[0], self.sfd, O.alpha(float(ah[0]), float(self.ad)), rows, H, I)
            work = 2.0 * rows * H * 2 * I + 2.0 * rows * I * H
        elif w == "grouped_swiglu":
            rows, H, I = self.rows, self.H, self.I
            qx, sfx = O.quantize(self.x, self.gx)
            ax = float(self.ax)
            gu_bits = O.gemm_gate_up_bf16(qx, self.qg, self.qu, sfx, self.sfg, self.sfu, O.alpha(ax, float(self.ag)),
                                          O.alpha(ax, float(self.au)), I, H, np.arange(rows)).reshape(1, rows, 2 * I)
            ah, gh = O.global_scale_batched(gu_bits, None, silu_mul=True)
            hq, hsf = O.silu_mul_quantize_batched(gu_bits, gh)
            O.gemm_ref(hq[0], self.qd, hsf[0], self.sfd, O.alpha(float(ah[0]), float(self.ad)), rows, H, I)
            work = 6.0 * rows * H * I
        elif w == "svdquant_linear":
            m, k, n = self.m, self.k, self.n
            xh = S.f32_to_bf16_bits(S.bf16_bits_to_f32(self.x) * S.bf16_bits_to_f32(self.pqs)[None, :])
            ax, gx = O.global_scale(xh)
            qx, sfx = O.quantize_smooth(self.x, self.pqs, gx)
            dd = O.lora_down(self.x, self.wd)
            d_bf16 = np.vectorize(O.f64_to_bf16, otypes=[np.uint16])(dd)
            al = O.alpha(float(ax), float(self.aw))
            l1 = S.f32_to_bf16_bits(self.l1_f32 / np.float32(al))
            O.gemm_ref(qx, self.qw, sfx, self.sfw, al, m, n, k, d=d_bf16, l1=l1, bias=self.bias)
            work = 2.0 * m * n * k + 2.0 * m * n * 64 + 2.0 * m * k * 64
        elif w == "pr1_linear":
            ax, gx = O.global_scale(self.x)
            qx, sfx = O.quantize(self.x, gx)
            O.gemm_ref(qx, self.qw, sfx, self.sfw, O.alpha(float(ax), float(self.aw)), 128, 256, 256)
            work = 2.0 * 128 * 256 * 256
        elif w in ("quant_dense", "quant_dense_fused"):
            a, g = O.global_scale(self.x)
            O.quantize(self.x, g)
            work = 2.5625 * self.x.size
        elif w in ("quant_masked", "quant_silu"):
            silu = w == "quant_silu"
            _, gs = O.global_scale_batched(self.x, None, silu_mul=silu)
            (O.silu_mul_quantize_batched if silu else O.quantize_masked_batched)(self.x, gs)
            work = (32704.0 if silu else 18368.0) * self.rows
        else:
            ax, gx = O.global_scale(self.x)
            qx, sfx = O.quantize(self.x, gx)
            O.gemm_ref(qx, self.qw, sfx, self.sfw, O.alpha(float(ax), float(self.aw)), self.m, self.n, self.k)
            work = 2.0 * self.m * self.n * self.k
        return work, time.perf_counter() - t0

    def measure(self, steps):
        work = secs = 0.0
        for _ in range(steps):
            w, dt = self.step()
            work += w
            secs += dt
        return scale(work / secs, self.unit), secs


# ---------------------------------------------------------------------------------------
# main
# ---------------------------------------------------------------------------------------

def run_reference(args, world, rank):
    if rank != 0:
        return       # the oracle runs on rank 0 only; the other ranks exit without work
    wl = args.workload
    rows = 1 if wl in ("swiglu_block", "grouped_swiglu") else None
    o = OracleSample(wl, rows)
    o.measure(args.warmup)
    t0 = time.perf_counter()
    value, secs = o.measure(args.steps)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": o.unit, "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / max(args.steps, 1),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64 (plain C oracle)",
            "data": "synthetic", "config": workload_config(wl, args.rank_lr, args.swiglu_path),
            "cpu_baseline": {"value": value, "unit": o.unit, "cores": o.threads, "kind": "oracle",
                             "sample": o.sample + " per step", **host_cpu()},
            "e2e": {"value": value, "unit": o.unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            "wall_s": round(time.perf_counter() - t0, 2)}
    print(json.dumps(line), flush=True)


# The other configurations, timed by the default run after the headline (one GPU only), each
# with its roofline and its oracle sample: (workload, low-rank r).
EXTRA_CONFIGS = [("pr1_linear", 0), ("quant_dense", 0), ("quant_masked", 0), ("quant_silu", 0),
                 ("grouped_moe", 0), ("lowrank", 32), ("lowrank", 64), ("lowrank", 128)]


class Timer:
    """CUDA-graph timing of one workload's step: a step graph (event nodes at its start and
    end only, kernels chained by programmatic dependent launch) and a kernel graph (an event
    node around every kernel), replayed alternately after an L2 flush."""

    def __init__(self, nv, wl, stream, flush_l2):
        import torch
        self.nv, self.wl, self.stream, self.flush_l2 = nv, wl, stream, flush_l2
        self.launches = launches = wl.launches()

        def step(evs=None):
            for i, (_, fn) in enumerate(launches):
                if evs is not None:
                    evs[i].record()
                fn()
            if evs is not None:
                evs[len(launches)].record()

        # One eager pass on the launch stream (allocates the library's per-stream scratch),
        # then the two CUDA graphs.  Should the CUDA driver refuse timing on graph event nodes,
        # every kernel is captured into its own graph and timed by events recorded around its
        # replay (no overlap either way).
        with torch.cuda.stream(stream):
            step()
        torch.cuda.synchronize()
        self.step_events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
        self.kernel_events = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(launches) + 1)]
        self.graph_s, self.graph_k = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph_s, stream=stream):
            self.step_events[0].record()
            step()
            self.step_events[1].record()
        with torch.cuda.graph(self.graph_k, stream=stream):
            step(self.kernel_events)
        torch.cuda.synchronize()
        self.mode = ("step: one CUDA graph per step, event nodes at its start and end (kernels chained by "
                     "programmatic dependent launch: %s); kernels: a second pass with an event node around every "
                     "kernel" % ("on" if nv.nvfp4_get_pdl() else "off"))
        self.split = None
        try:
            with torch.cuda.stream(stream):
                self.run_step()
                self.run_kernels()
        except Exception:                                      # noqa: BLE001
            torch.cuda.synchronize()
            self.graph_s = self.graph_k = None
            self.split = []
            for _, fn in launches:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g, stream=stream):
                    fn()
                self.split.append(g)
            self.outer = [torch.cuda.Event(enable_timing=True) for _ in range(len(launches) + 1)]
            self.mode = "one CUDA graph per kernel, events around each replay (step time = first to last event)"

    def replay_step(self):
        if self.split is None:
            self.graph_s.replay()
        else:
            for g in self.split:
                g.replay()

    def run_kernels(self):
        if self.split is None:
            self.graph_k.replay()
            self.stream.synchronize()
            ev = self.kernel_events
        else:
            for i, g in enumerate(self.split):
                self.outer[i].record()
                g.replay()
            self.outer[-1].record()
            self.stream.synchronize()
            ev = self.outer
        return [ev[i].elapsed_time(ev[i + 1]) for i in range(len(self.launches))]

    def run_step(self):
        if self.split is not None:
            self.run_kernels()
            return self.outer[0].elapsed_time(self.outer[-1])
        self.graph_s.replay()
        self.stream.synchronize()
        return self.step_events[0].elapsed_time(self.step_events[1])

    def warm(self, n):
        import torch
        with torch.cuda.stream(self.stream):
            for _ in range(n):
                self.flush_l2()
                self.replay_step()
        torch.cuda.synchronize()

    def timed(self, steps):
        """`steps` replays of each graph, alternating step by step, so that both passes see the
        same clocks and power state.  Returns (step times, per-step kernel times) in ms."""
        import torch
        step_ms, samples = [], []
        with torch.cuda.stream(self.stream):
            for _ in range(steps):
                self.flush_l2()
                step_ms.append(self.run_step())
                self.flush_l2()
                samples.append(self.run_kernels())
        torch.cuda.synchronize()
        return step_ms, samples

    def release(self):
        self.graph_s = self.graph_k = self.split = None


def summarize(wl, step_ms, samples, launches, peaks, peak_kind, world):
    """value / ms_per_step (whole job), per-kernel parts and the dominant kernel's roofline."""
    per_kernel = {name: [smp[i] for smp in samples] for i, (name, _) in enumerate(launches)}
    steps = len(step_ms)
    work_all, total_ms_max = aggregate(world, wl.work() * steps, sum(step_ms))
    value = scale(work_all / (total_ms_max * 1e-3), wl.unit)
    fp4_peak = peaks["bf16_tflops"] * FP4_OVER_BF16
    hbm_peak = peaks["hbm_gbs"]
    parts = {}
    for name, (w, unit) in wl.kernel_work().items():
        ms = statistics.mean(per_kernel[name])
        ach = scale(w / (ms * 1e-3), unit)
        peak = fp4_peak if unit == "TFLOP/s" else hbm_peak
        parts[name] = {"ms": round(ms, 5), "achieved": round(ach, 2), "unit": unit, "frac": round(ach / peak, 4)}
    dom = wl.dominant
    w, unit = wl.kernel_work()[dom]
    dom_ms = statistics.mean(per_kernel[dom])
    achieved = scale(w / (dom_ms * 1e-3), unit)
    peak = fp4_peak if unit == "TFLOP/s" else hbm_peak
    kernel_name = KERNEL_OF_LAUNCH.get(dom, "nvfp4_gemm_kernel" if unit == "TFLOP/s" else "quantize_kernel")
    roofline = {"bound": "tensor" if unit == "TFLOP/s" else "hbm", "achieved": round(achieved, 2),
                "peak": round(peak, 1), "unit": unit, "frac": round(achieved / peak, 4),
                "traffic": recorded_traffic(kernel_name, f"{wl.name}:{dom}"), "kernel": dom,
                "peak_source": f"{peak_kind}: " + (
                    f"bf16 burst {peaks['bf16_tflops']} TFLOP/s x {FP4_OVER_BF16} (nominal FP4/BF16 dense ratio)"
                    if unit == "TFLOP/s" else f"HBM copy {peaks['hbm_gbs']} GB/s")}
    return value, total_ms_max / steps, parts, roofline


def measure_e2e(wl, timer, stream, flush_l2, args, world):
    """End to end through the public API: every step uploads its input from pinned host
    memory and downloads its result.  Uploads, compute and downloads run on three streams
    (PCIe is full duplex), through double-buffered device staging tensors ordered by events,
    so step i+1 uploads and step i-1 downloads while step i computes."""
    import torch
    x_host_bits, x_dev, y_dev = wl.e2e_io()
    x_pinned = torch.from_numpy(np.ascontiguousarray(x_host_bits).view(np.int16)).view(x_dev.dtype).pin_memory()
    y_pinned = [torch.empty(y_dev.shape, dtype=y_dev.dtype).pin_memory() for _ in range(2)]
    x_stage = [torch.empty_like(x_dev) for _ in range(2)]
    y_stage = [torch.empty_like(y_dev) for _ in range(2)]
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    total = args.warmup + args.steps
    ev_in, ev_used, ev_out, ev_down = ([torch.cuda.Event() for _ in range(total)] for _ in range(4))
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    for i in range(total):
        buf = i % 2
        with torch.cuda.stream(h2d):
            if i == args.warmup:
                t_start.record()
            if i >= 2:
                h2d.wait_event(ev_used[i - 2])          # staging buffer free again
            x_stage[buf].copy_(x_pinned, non_blocking=True)
            ev_in[i].record()
        with torch.cuda.stream(stream):
            flush_l2()
            stream.wait_event(ev_in[i])
            x_dev.copy_(x_stage[buf], non_blocking=True)
            ev_used[i].record()
            timer.replay_step()
            if i >= 2:
                stream.wait_event(ev_down[i - 2])
            y_stage[buf].copy_(y_dev, non_blocking=True)
            ev_out[i].record()
        with torch.cuda.stream(d2h):
            d2h.wait_event(ev_out[i])
            y_pinned[buf].copy_(y_stage[buf], non_blocking=True)
            ev_down[i].record()
    with torch.cuda.stream(d2h):
        t_end.record()
    torch.cuda.synchronize()
    e2e_ms = t_start.elapsed_time(t_end)
    e2e_work, e2e_ms = aggregate(world, wl.work() * args.steps, e2e_ms)
    e2e_val = scale(e2e_work / (e2e_ms * 1e-3), wl.unit)
    return {"value": round(e2e_val, 3), "unit": wl.unit,
            "h2d_bytes_per_step": int(x_pinned.numel() * x_pinned.element_size()),
            "d2h_bytes_per_step": int(y_pinned[0].numel() * y_pinned[0].element_size()),
            "ms_per_step": round(e2e_ms / args.steps, 4),
            "pipeline": "upload, compute and download on three streams, double-buffered device staging; time from "
                        "the first timed upload to the last timed download"}


def measure_sustained(timer, wl, world, local, min_seconds=1.0):
    """The step graph replayed back to back (each replay after an L2 flush) for at least
    `min_seconds` of wall time: the power-capped regime a long run settles in, with its own
    clock record."""
    import torch
    step_ms = []
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t0 = time.perf_counter()
        with torch.cuda.stream(timer.stream):
            while time.perf_counter() - t0 < min_seconds:
                timer.flush_l2()
                step_ms.append(timer.run_step())
        torch.cuda.synchronize()
        wall = time.perf_counter() - t0
    barrier(world)
    work_all, total_ms_max = aggregate(world, wl.work() * len(step_ms), sum(step_ms))
    clk = clocks.summary()
    return {"value": round(scale(work_all / (total_ms_max * 1e-3), wl.unit), 3), "unit": wl.unit,
            "ms_per_step": round(total_ms_max / len(step_ms), 5), "steps": len(step_ms), "wall_s": round(wall, 3),
            "clocks": {"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                       "reasons": clk.get("reasons"), "power_w_max": clk.get("power_w_max")}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="nvfp4", choices=["nvfp4", "reference"])
    ap.add_argument("--workload", default="swiglu_block",
                    choices=["swiglu_block", "quant_dense", "quant_dense_fused", "quant_masked", "quant_silu", "grouped_moe",
                             "grouped_swiglu", "lowrank", "svdquant_linear", "pr1_linear", "bf16a_linear"])
    ap.add_argument("--rank-lr", type=int, default=64)
    ap.add_argument("--swiglu-path", default="fused", choices=["fused", "unfused"],
                    help="swiglu_block: SiLU*mul quantization in the gate/up GEMM epilogue, or as its own kernel")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="time only the chosen workload (the default run also times the other configurations)")
    ap.add_argument("--no-sustained", action="store_true")
    ap.add_argument("--no-pdl", action="store_true",
                    help="launch without programmatic dependent launch (the library default is on)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    if args.impl == "reference":
        world = int(os.environ.get("WORLD_SIZE", "1"))
        rank = int(os.environ.get("RANK", "0"))
        run_reference(args, world, rank)
        return

    import torch
    import nvfp4_block_scaled_16_b200 as nv
    world, rank, local = dist_setup(args.gpus)
    nv.load_library()
    if args.no_pdl:
        nv.nvfp4_set_pdl(False)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device="cuda")
    clean = torch.ones(L2_CLEAN_BYTES // 4, dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def flush_l2():
        flush.zero_()
        clean.max()

    peaks, peak_kind = load_peaks()
    wl = make_workload(args.workload, nv, args.rank_lr, args.swiglu_path)
    timer = Timer(nv, wl, stream, flush_l2)
    timer.warm(args.warmup)
    if nv.nvfp4_device_status(clear=True) != 0:
        raise SystemExit("device-side timeout during warm-up")

    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(local) as clocks:
        t_wall = time.perf_counter()
        step_ms, samples = timer.timed(args.steps)
        t_wall = time.perf_counter() - t_wall
    clk = clocks.summary()
    barrier(world)
    status = nv.nvfp4_device_status(clear=True)
    if status != 0:
        raise SystemExit(f"device-side timeout in the timed region (status {status})")
    value, ms_per_step, parts, roofline = summarize(wl, step_ms, samples, timer.launches, peaks, peak_kind, world)

    sustained = None if args.no_sustained else measure_sustained(timer, wl, world, local)
    e2e = None
    if not args.no_e2e and wl.e2e_io() is not None:
        e2e = measure_e2e(wl, timer, stream, flush_l2, args, world)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        o = OracleSample(wl.name)
        v, secs = o.measure(1)
        cpu = {"value": v, "unit": wl.unit, "cores": o.threads, "kind": "oracle", "sample": o.sample,
               "seconds": round(secs, 2), **host_cpu()}
    n_launches = 2 * len(timer.launches) * args.steps
    unit, config, timing_mode = wl.unit, wl.config(), timer.mode
    timer.release()
    del timer, wl
    torch.cuda.synchronize()
    torch.cuda.empty_cache()

    # the other configurations (one GPU: the scaling runs time the headline only)
    configs = None
    if world == 1 and not args.no_configs and args.workload == "swiglu_block":
        configs = {}
        for name, r in EXTRA_CONFIGS:
            key = f"{name}_r{r}" if name == "lowrank" else name
            w = make_workload(name, nv, r or args.rank_lr)
            t = Timer(nv, w, stream, flush_l2)
            t.warm(args.warmup)
            with ClockSampler(local) as ck:
                sm, smp = t.timed(args.steps)
            st = nv.nvfp4_device_status(clear=True)
            if st != 0:
                raise SystemExit(f"device-side timeout while timing {key} (status {st})")
            v, ms, prt, rl = summarize(w, sm, smp, t.launches, peaks, peak_kind, world)
            n_launches += 2 * len(t.launches) * args.steps
            entry = {"value": round(v, 3), "unit": w.unit, "ms_per_step": round(ms, 5), "roofline": rl, "parts": prt,
                     "config": w.config(), "clocks": {k: ck.summary().get(k) for k in ("sm_mhz", "reasons")}}
            if not args.no_cpu_baseline:
                o = OracleSample(name)
                cv, secs = o.measure(1)
                entry["cpu_baseline"] = {"value": cv, "unit": o.unit, "cores": o.threads, "kind": "oracle",
                                         "sample": o.sample, "seconds": round(secs, 2)}
            configs[key] = entry
            t.release()
            del t, w
            torch.cuda.synchronize()
            torch.cuda.empty_cache()

    if rank == 0:
        line = {"metric": METRIC, "value": round(value, 3), "unit": unit, "n_gpus": world,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
                "dtype": "e2m1 x e2m1 (ue4m3 block scales) -> f32 accumulate",
                "data": "synthetic (seeded N(0,1) activations, N(0,0.02) weights)", "config": config,
                "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
                # our kernels launched in the timed regions: the step pass and the kernel pass of
                # the headline and of every other configuration
                "gpu_launches": n_launches, "parts": parts,
                "clocks": {"sm_mhz": clk.get("sm_mhz"), "sm_max_mhz": clk.get("sm_max_mhz"),
                           "reasons": clk.get("reasons")},
                "sustained": sustained, "configs": configs,
                "wall_s_timed_region": round(t_wall, 4), "timing": timing_mode}
        if world > 1:
            line["config"]["parallelism"] = f"dp{world} (independent batch per GPU, no collective)"
        print(json.dumps(line), flush=True)

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
