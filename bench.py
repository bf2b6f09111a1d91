"""Benchmark of the block-scaled FP8 hot path on B200.

One step (default workload `moe_grouped`, the largest single-GPU case) =
the expert up-projection of an MoE layer: 16384 bf16 tokens x 7168 routed
top-8 over 64 experts; the FP8 dispatch (route histograms and scan, layout,
one fused kernel that quantizes each token row once to MXFP8 and writes it
to the rows of its 8 experts) builds the expert-grouped operand [131072,
7168], and the grouped MXFP8 GEMM multiplies it with the prequantized expert
weights 64 x [2048, 7168], fp32 accumulation, bf16 out (3.848 TFLOP).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
                    [--workload moe_grouped|ds_fp8_gemm|qat_forward|qat_backward|moe_dispatch|
                                moe_prequant|nvfp4_gemm|dequant]

Prints one JSON line (rank 0).  `value` is whole-step throughput in TFLOP/s
(GEMM flops of the step / step time, quantization included; GB/s for the
quantize-, dequantize- and dispatch-only workloads), with the inputs
resident in HBM and L2 flushed (256 MiB write) before every step; the
per-kernel times, the quantize GB/s and the roofline of the dominant kernel
come from CUDA events on the launching stream.  With N > 1 (torchrun) every
rank runs an independent replica (the path has no exchange step): the time
is the max over ranks and `value` counts all ranks' work.  `cpu_baseline`
is the oracle timed on a bounded sample, on one thread and on every host
core; `--impl reference` times the oracle alone (every host core), one
sample of the workload per step.
"""
from __future__ import annotations

import argparse
import glob
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads  # noqa: E402

FLUSH_BYTES = 256 << 20


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while running."""

    REASONS = {0x8: "hw_slowdown", 0x40: "hw_thermal_slowdown", 0x20: "sw_thermal_slowdown",
               0x4: "sw_power_cap", 0x80: "hw_power_brake_slowdown", 0x1: "gpu_idle",
               0x2: "applications_clocks_setting", 0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self._nv.nvmlDeviceGetClockInfo(self._h, self._nv.NVML_CLOCK_SM))
                r = self._nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for bit, name in self.REASONS.items():
                    if r & bit and name != "gpu_idle":
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.002)

    def __enter__(self):
        if self._nv:
            self._t.start()
        return self

    def __exit__(self, *a):
        self._stop.set()
        if self._nv:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples),
                "source": "nvml" if self._nv else "unavailable"}


# ------------------------------------------------------------------ workloads on the GPU

class Step:
    """A workload bound to device buffers; run() enqueues one step."""
    name = ""
    CONFIG: dict = {}          # the workload's description and shape (both bench arms print it)
    flops = 0.0
    quant_bytes = 0.0
    launches = 0
    dominant = ""
    unit = "TFLOP/s"           # the rate `value` is reported in: flops (GEMM steps) or bytes
    dtype = "e4m3xe4m3->f32 (bf16 in/out)"
    tensor_ratio = 2.0         # the GEMM's dense tensor peak / the measured bf16 peak (nominal 4.5 / 2.25)

    @property
    def work(self) -> float:
        """Work of one step in the unit's numerator (flops, or bytes for GB/s)."""
        return self.flops

    # kernels that depend on nothing earlier in the step and run on a second
    # stream in the timed step, joined back before `join_before`
    side = ()
    join_before = ""

    def kernels(self):  # list of (label, callable)
        raise NotImplementedError

    # Device tensors (attribute names) a step copies in from pinned host
    # memory and reads back, for the pipelined end-to-end loop; empty: the
    # workload has only the one-step-after-another loop (e2e_step).
    E2E_IN: tuple = ()
    E2E_OUT: tuple = ()

    def e2e_pipelined(self, steps: int, side_stream):
        """The steps as a serving loop runs them: two slots of the step's
        device inputs and outputs, so that the upload of step i + 1 (a copy
        stream) and the readback of step i - 1 (a second copy stream) overlap
        the kernels of step i.  Every step still copies all of its inputs from
        pinned host memory and reads its whole output back.  Returns (ms per
        step, H2D bytes per step, D2H bytes per step)."""
        names = self.E2E_IN + self.E2E_OUT
        if not hasattr(self, "_e2e_host"):
            self._e2e_host = {n: getattr(self, n).cpu().pin_memory() for n in names}
            self._e2e_slot1 = {n: torch.empty_like(getattr(self, n)) for n in names}
        slots = [{n: getattr(self, n) for n in names}, self._e2e_slot1]
        host = self._e2e_host
        up, down, comp = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.current_stream()
        loaded, computed, drained = ([torch.cuda.Event(), torch.cuda.Event()] for _ in range(3))
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        saved = dict(slots[0])
        torch.cuda.synchronize()
        t0.record(comp)
        up.wait_stream(comp)
        down.wait_stream(comp)
        for i in range(steps):
            k = i % 2
            with torch.cuda.stream(up):
                if i >= 2:
                    up.wait_event(computed[k])          # slot k's inputs were read by step i - 2
                for n in self.E2E_IN:
                    slots[k][n].copy_(host[n], non_blocking=True)
                loaded[k].record(up)
            comp.wait_event(loaded[k])
            if i >= 2:
                comp.wait_event(drained[k])             # slot k's outputs were read back after step i - 2
            for n in names:
                setattr(self, n, slots[k][n])
            self.whole_step(side_stream)
            computed[k].record(comp)
            with torch.cuda.stream(down):
                down.wait_event(computed[k])
                for n in self.E2E_OUT:
                    host[n].copy_(slots[k][n], non_blocking=True)
                drained[k].record(down)
        comp.wait_stream(up)
        comp.wait_stream(down)
        t1.record(comp)
        t1.synchronize()
        for n, t in saved.items():
            setattr(self, n, t)
        nbytes = lambda ns: sum(host[n].numel() * host[n].element_size() for n in ns)
        return t0.elapsed_time(t1) / steps, nbytes(self.E2E_IN), nbytes(self.E2E_OUT)

    def whole_step(self, side_stream):
        """One step as the timed graph and the end-to-end loop run it: the
        kernels named in `side` on `side_stream`, forked from the current
        stream before the step's first kernel (so they run beside the kernels
        listed before `join_before`, not after them), the rest in order on
        the current stream, which waits for the side stream before
        `join_before`."""
        cur = torch.cuda.current_stream()
        joined = not self.side
        if self.side:
            side_stream.wait_stream(cur)              # the step's inputs are ready on both streams
        for name, fn in self.kernels():
            if name in self.side:
                with torch.cuda.stream(side_stream):
                    fn()
                continue
            if not joined and name == self.join_before:
                cur.wait_stream(side_stream)
                joined = True
            fn()
        if not joined:
            cur.wait_stream(side_stream)


class DsFp8Gemm(Step):
    name = "ds_fp8_gemm"
    E2E_IN, E2E_OUT = ("a", "b"), ("c",)
    CONFIG = {"workload": "ds_fp8_gemm: A bf16 4096x7168 N(0,1) -> E4M3 with fp32 scale per 1x128 tile; "
                          "B bf16 2048x7168 N(0,0.02) -> E4M3 with fp32 scale per 128x128 block; "
                          "C = A B^T fp32 accumulate, bf16 out",
              "m": 4096, "n": 2048, "k": 7168, "l2": "flushed before every step (256 MiB write)"}
    dominant = "gemm_fp8_f32scale"
    side = ("quant_fp8_128x128",)      # B's quantizer runs beside A's
    join_before = "gemm_fp8_f32scale"

    def __init__(self, fpq, dev, m=4096, n=2048, k=7168):
        self.f = fpq
        self.m, self.n, self.k = m, n, k
        wl = workloads.ds_fp8_gemm(m, n, k)
        self.a_host, self.b_host = wl["a"].pin_memory(), wl["b"].pin_memory()
        self.a, self.b = self.a_host.to(dev), self.b_host.to(dev)
        f = fpq
        self.qa = torch.empty((m, k), dtype=torch.uint8, device=dev)
        self.sa = torch.empty((m, k // 128), dtype=torch.float32, device=dev)
        self.qb = torch.empty((n, k), dtype=torch.uint8, device=dev)
        self.sb = torch.empty(((n + 127) // 128, k // 128), dtype=torch.float32, device=dev)
        self.c = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        self.c_host = torch.empty((m, n), dtype=torch.bfloat16).pin_memory()
        self.flops = 2.0 * m * n * k
        self.qa_bytes = m * k * (2 + 1) + m * (k // 128) * 4
        self.qb_bytes = n * k * (2 + 1) + ((n + 127) // 128) * (k // 128) * 4
        self.quant_bytes = self.qa_bytes + self.qb_bytes
        self.launches = 3
        self.config = dict(self.CONFIG)

    def kernels(self):
        f = self.f
        return [
            ("quant_fp8_1x128", lambda: f.fpq_quantize_block(f.FP8_1x128, self.a, 1, self.m, self.k, self.qa, self.sa)),
            ("quant_fp8_128x128", lambda: f.fpq_quantize_block(f.FP8_128x128, self.b, 1, self.n, self.k, self.qb, self.sb)),
            ("gemm_fp8_f32scale", lambda: f.fpq_scaled_gemm(f.FP8_1x128, self.qa, self.sa, f.FP8_128x128, self.qb,
                                                            self.sb, self.m, self.n, self.k, self.c, f.OUT_BF16)),
        ]

    def kernel_work(self):
        return {"quant_fp8_1x128": ("GB/s", self.qa_bytes), "quant_fp8_128x128": ("GB/s", self.qb_bytes),
                "gemm_fp8_f32scale": ("TFLOP/s", self.flops)}

    def e2e_step(self, stream, side_stream):
        """Host buffers in, host buffer out: the same step through the C ABI
        with the copies inside the timed region."""
        self.a.copy_(self.a_host, non_blocking=True)
        self.b.copy_(self.b_host, non_blocking=True)
        self.whole_step(side_stream)
        self.c_host.copy_(self.c, non_blocking=True)
        return self.a_host.numel() * 2 + self.b_host.numel() * 2, self.c.numel() * 2


class MoeGrouped(Step):
    """The expert up-projection of an MoE layer on one GPU: 16384 bf16
    tokens x 7168, top-8 of 64 experts.  The FP8 dispatch (route, layout, and
    the fused kernel that quantizes each token row once to MXFP8 and writes
    it to the rows of its 8 experts) builds the expert-grouped operand; the
    grouped MXFP8 GEMM multiplies it with the prequantized expert weights
    64 x 2048 x 7168."""
    name = "moe_grouped"
    dominant = "gemm_grouped_mxfp8"
    E2E_IN, E2E_OUT = ("x", "ids"), ("c",)
    CONFIG = {"workload": "moe_grouped: X 16384x7168 N(0,1), top-8 of 64 experts (Zipf 1.1 Gumbel-top-8); "
                          "FP8 dispatch (each token quantized once to MXFP8, 131072 rows grouped by "
                          "expert); grouped GEMM with MXFP8 expert weights 64x2048x7168", "l2": "flushed before every step (256 MiB write)"}

    def __init__(self, fpq, dev, tokens=16384, experts=64, topk=8):
        self.f = fpq
        wl = workloads.moe_grouped()
        self.x_host = wl["x"].pin_memory()
        self.ids_host = workloads.route_choices(tokens, experts, topk, seed=5001).pin_memory()
        self.x, self.ids = self.x_host.to(dev), self.ids_host.to(dev)
        self.w = wl["w"].to(dev)
        self.wq, self.ws = fpq.quantize(self.w, fpq.MXFP8)      # weights are prequantized once (serving)
        del self.w
        self.tokens, self.k = self.x.shape
        self.topk, self.e = topk, experts
        self.total = tokens * topk
        self.groups, self.n = self.wq.shape[0], self.wq.shape[1]
        i32, i64, u8 = (dict(dtype=d, device=dev) for d in (torch.int32, torch.int64, torch.uint8))
        self.counts_dev = torch.empty((experts,), **i32)
        wsb = fpq.fpq_moe_route_workspace_bytes(tokens, experts)
        self.rws = torch.empty(((wsb + 15) // 16 * 16,), **u8)
        self.row0 = torch.empty((experts,), **i64)
        self.offsets = torch.empty((experts + 1,), **i32)
        self.qx = torch.empty((self.total, self.k), **u8)
        self.sx = torch.empty((self.total, self.k // 32), **u8)
        self.qp = torch.tensor([self.qx.data_ptr()], **i64)
        self.sp = torch.tensor([self.sx.data_ptr()], **i64)
        self.cap = torch.tensor([self.total], **i64)
        self.c = torch.empty((self.total, self.n), dtype=torch.bfloat16, device=dev)
        self.c_host = torch.empty(self.c.shape, dtype=self.c.dtype).pin_memory()
        self.flops = 2.0 * self.total * self.n * self.k
        self.route_bytes = self.total * 4
        self.dispatch_bytes = self.tokens * self.k * 2 + self.total * 4 + self.total * (self.k + self.k // 32)
        self.quant_bytes = self.route_bytes + self.dispatch_bytes
        self.launches = 5
        counts = np.bincount(self.ids_host.numpy().reshape(-1), minlength=experts)
        self.config = dict(self.CONFIG, expert_rows_max=int(counts.max()), expert_rows_min=int(counts.min()))

    def kernels(self):
        f = self.f
        return [
            ("moe_route", lambda: f.fpq_moe_route(self.ids, self.tokens, self.topk, self.e, self.counts_dev,
                                                  self.rws)),
            ("moe_layout", lambda: f.fpq_moe_dispatch_layout(self.counts_dev, 1, self.e, 0, f.MOE_DIRECT, self.row0,
                                                             self.offsets)),
            ("moe_dispatch_mxfp8", lambda: f.fpq_moe_dispatch_mxfp8(self.x, self.tokens, self.k, self.ids, self.topk,
                                                                    self.e, self.rws, self.row0, 1, self.qp, self.sp,
                                                                    self.cap)),
            ("gemm_grouped_mxfp8", lambda: f.fpq_grouped_scaled_gemm(f.MXFP8, self.qx, self.sx, self.wq, self.ws,
                                                                     self.offsets, self.groups, self.total, self.n,
                                                                     self.k, self.c, f.OUT_BF16)),
        ]

    def kernel_work(self):
        return {"moe_route": ("GB/s", self.route_bytes), "moe_layout": ("GB/s", self.e * 8),
                "moe_dispatch_mxfp8": ("GB/s", self.dispatch_bytes), "gemm_grouped_mxfp8": ("TFLOP/s", self.flops)}

    def e2e_step(self, stream, side_stream):
        """Tokens and their routing from pinned host memory in, the expert
        outputs back to pinned host memory, copies inside the timed region
        (the expert weights stay resident: serving)."""
        self.x.copy_(self.x_host, non_blocking=True)
        self.ids.copy_(self.ids_host, non_blocking=True)
        self.whole_step(side_stream)
        self.c_host.copy_(self.c, non_blocking=True)
        return self.x_host.numel() * 2 + self.ids_host.numel() * 4, self.c.numel() * 2


class QatForward(Step):
    name = "qat_forward"
    E2E_IN, E2E_OUT = ("w", "la", "lb", "x"), ("c",)
    dominant = "gemm_fp8_f32scale"
    CONFIG = {"workload": "qat_forward: merge W 2048x7168 + (32/16) B A (r=16) -> 128x128 FP8 fake-quant; "
                          "X 8192x7168 -> 1x128 FP8; C = X W_eff^T", "l2": "flushed before every step (256 MiB write)"}
    side = ("lora_merge_fq",)          # the weight merge runs beside X's quantizer
    join_before = "gemm_fp8_f32scale"

    def __init__(self, fpq, dev):
        self.f = fpq
        wl = workloads.qat_forward()
        self.w, self.la, self.lb, self.x = (wl[t].to(dev) for t in ("w", "lora_a", "lora_b", "x"))
        self.aor = wl["alpha_over_r"]
        self.n, self.k = self.w.shape
        self.m = self.x.shape[0]
        self.wq = torch.empty((self.n, self.k), dtype=torch.uint8, device=dev)
        self.ws = torch.empty((self.n // 128, self.k // 128), dtype=torch.float32, device=dev)
        self.xq = torch.empty((self.m, self.k), dtype=torch.uint8, device=dev)
        self.xs = torch.empty((self.m, self.k // 128), dtype=torch.float32, device=dev)
        self.c = torch.empty((self.m, self.n), dtype=torch.bfloat16, device=dev)
        self.flops = 2.0 * self.m * self.n * self.k
        self.merge_bytes = self.n * self.k * 3 + (self.la.numel() + self.lb.numel()) * 2
        self.xq_bytes = self.m * self.k * 3 + self.m * (self.k // 128) * 4
        self.quant_bytes = self.merge_bytes + self.xq_bytes
        self.launches = 3
        self.config = dict(self.CONFIG)

    def kernels(self):
        f = self.f
        return [
            ("lora_merge_fq", lambda: f.fpq_lora_merge_fakequant(self.w, self.la, self.lb, self.n, self.k, 16, self.aor,
                                                                 self.wq, self.ws)),
            ("quant_fp8_1x128", lambda: f.fpq_quantize_block(f.FP8_1x128, self.x, 1, self.m, self.k, self.xq, self.xs)),
            ("gemm_fp8_f32scale", lambda: f.fpq_scaled_gemm(f.FP8_1x128, self.xq, self.xs, f.FP8_128x128, self.wq,
                                                            self.ws, self.m, self.n, self.k, self.c, f.OUT_BF16)),
        ]

    def kernel_work(self):
        return {"lora_merge_fq": ("GB/s", self.merge_bytes), "quant_fp8_1x128": ("GB/s", self.xq_bytes),
                "gemm_fp8_f32scale": ("TFLOP/s", self.flops)}

    def e2e_step(self, stream, side_stream):
        """Base weight, LoRA factors and activations from pinned host memory
        in, the GEMM output back to pinned host memory, copies inside the
        timed region."""
        if not hasattr(self, "host"):
            self.host = [t.cpu().pin_memory() for t in (self.w, self.la, self.lb, self.x)]
            self.c_host = torch.empty(self.c.shape, dtype=self.c.dtype).pin_memory()
        for d, h in zip((self.w, self.la, self.lb, self.x), self.host):
            d.copy_(h, non_blocking=True)
        self.whole_step(side_stream)
        self.c_host.copy_(self.c, non_blocking=True)
        return sum(h.numel() * 2 for h in self.host), self.c.numel() * 2


class MoePrequant(Step):
    """MoE expert prequantization: 64 experts x {gate, up [2048, 7168]; down
    [7168, 2048]} bf16 N(0, 0.02), each projection's 64 matrices quantized by
    one batched call, to MXFP8 (1x32, E8M0) and to NVFP4 (1x16 E4M3 + a
    per-matrix fp32 scale).  The step's work is the algorithmic bytes."""
    name = "moe_prequant"
    CONFIG = {"workload": "moe_prequant: 64 experts x {gate, up 2048x7168; down 7168x2048} bf16 N(0,0.02) "
                          "-> MXFP8 (1x32 E8M0) and NVFP4 (1x16 E4M3 + fp32 per matrix); one batched call "
                          "per projection and format", "l2": "flushed before every step (256 MiB write)"}
    side = ("quant_nvfp4",)            # the two formats of a matrix are independent
    dominant = "quant_nvfp4"
    unit = "GB/s"
    dtype = "bf16 -> e4m3 / e2m1 codes (fp32 scale arithmetic)"

    def __init__(self, fpq, dev, experts=64):
        self.f = fpq
        self.e = experts
        shapes = {"gate": (2048, 7168), "up": (2048, 7168), "down": (7168, 2048)}
        self.x, self.mx, self.nv, self.host = {}, {}, {}, {}
        for i, (nm, (r, c)) in enumerate(shapes.items()):
            g = torch.Generator(device=dev)
            g.manual_seed(4000 + i)
            x = torch.empty((experts, r, c), dtype=torch.bfloat16, device=dev)
            for e in range(experts):
                x[e] = (torch.randn(r, c, generator=g, device=dev) * 0.02).to(torch.bfloat16)
            self.x[nm] = (x, r, c)
            self.mx[nm] = (torch.empty((experts, r, c), dtype=torch.uint8, device=dev),
                           torch.empty((experts, r, c // 32), dtype=torch.uint8, device=dev))
            wsb = fpq.fpq_quantize_workspace_bytes(fpq.NVFP4, experts)
            self.nv[nm] = (torch.empty((experts, r, c // 2), dtype=torch.uint8, device=dev),
                           torch.empty((experts, r, c // 16), dtype=torch.uint8, device=dev),
                           torch.empty((experts,), dtype=torch.float32, device=dev),
                           torch.empty(((wsb + 15) // 16 * 16,), dtype=torch.uint8, device=dev))
        elems = sum(experts * r * c for _, r, c in self.x.values())
        self.mx_bytes = elems * (2 + 1 + 1 / 32)
        self.nv_bytes = elems * (2 + 0.5 + 1 / 16) + 4 * 3 * experts
        self.quant_bytes = self.mx_bytes + self.nv_bytes
        self.launches = 6
        self.config = dict(self.CONFIG, elements=elems)
        if experts != 64:
            self.config["workload"] = self.CONFIG["workload"].replace("64 experts", f"{experts} experts")

    @property
    def work(self) -> float:
        return self.quant_bytes

    def kernels(self):
        f = self.f

        def mx():
            for nm, (x, r, c) in self.x.items():
                q, s_ = self.mx[nm]
                f.fpq_quantize_block(f.MXFP8, x, self.e, r, c, q, s_)

        def nv():
            for nm, (x, r, c) in self.x.items():
                q, s_, g, ws = self.nv[nm]
                f.fpq_quantize_block(f.NVFP4, x, self.e, r, c, q, s_, g, ws)

        return [("quant_mxfp8", mx), ("quant_nvfp4", nv)]

    def kernel_work(self):
        return {"quant_mxfp8": ("GB/s", self.mx_bytes), "quant_nvfp4": ("GB/s", self.nv_bytes)}

    def e2e_step(self, stream, side_stream):
        """bf16 expert stacks in pinned host memory in, every code and scale
        back to pinned host memory, copies inside the timed region."""
        if not self.host:
            for nm, (x, r, c) in self.x.items():
                outs = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (*self.mx[nm], *self.nv[nm][:3])]
                self.host[nm] = (x.cpu().pin_memory(), outs)
        hb = db = 0
        for nm, (x, r, c) in self.x.items():
            x.copy_(self.host[nm][0], non_blocking=True)
            hb += x.numel() * 2
        for _, fn in self.kernels():
            fn()
        for nm in self.x:
            for h, d in zip(self.host[nm][1], (*self.mx[nm], *self.nv[nm][:3])):
                h.copy_(d, non_blocking=True)
                db += d.numel() * d.element_size()
        return hb, db


class QatBackward(Step):
    """The backward of the QAT linear layer (straight-through estimator) at
    the QAT workload's shape: x 8192x7168, W 2048x7168, LoRA r = 16, alpha/r
    = 2; dx, dW_eff, dA, dB in bf16 on the bf16 tensor-core GEMM, each
    operand read in its stored layout; dA and dB from one pass over dW (each
    dW tile feeds both products) plus an ordered reduction of the partial
    sums.  The same launches as fpq_qat_backward, issued through the C ABI
    one by one so that each product is timed."""
    name = "qat_backward"
    dominant = "gemm_bf16_dx"
    CONFIG = {"workload": "qat_backward: dy 8192x2048 N(0,1); x_fq = 1x128 fake-quant of x 8192x7168 "
                          "N(0,1); w_fq = 128x128 fake-quant of W + 2 B A (W 2048x7168 N(0,0.02), r = 16); "
                          "dx = dy w_fq, dW = dy^T x_fq, dA = 2 B^T dW, dB = 2 dW A^T, bf16",
              "m": 8192, "n": 2048, "k": 7168, "r": 16, "l2": "flushed before every step (256 MiB write)"}
    dtype = "bf16xbf16->f32 (bf16 out)"
    tensor_ratio = 1.0

    def __init__(self, fpq, dev, m=8192, n=2048, k=7168):
        self.f = fpq
        wl = workloads.qat_forward(m=m, n=n, k=k)
        r = wl["lora_a"].shape[0]
        self.m, self.n, self.k, self.r = m, n, k, r
        self.aor = wl["alpha_over_r"]
        x, w = wl["x"].to(dev), wl["w"].to(dev)
        self.a, self.b = wl["lora_a"].to(dev), wl["lora_b"].to(dev)
        # the forward's fake-quantized operands, made by the library
        xq, xs = fpq.quantize(x, fpq.FP8_1x128)
        self.x_fq = fpq.dequantize(fpq.FP8_1x128, xq, xs)
        self.w_fq = fpq.lora_merge_fakequant(w, self.a, self.b, self.aor, want_fq=True)[2]
        del x, w, xq, xs
        self.dy_host = workloads.normal_bf16((m, n), 1.0, seed=3005).pin_memory()
        self.dy = self.dy_host.to(dev)
        bf = dict(dtype=torch.bfloat16, device=dev)
        self.dx, self.dw = torch.empty((m, k), **bf), torch.empty((n, k), **bf)
        self.da, self.db = torch.empty((r, k), **bf), torch.empty((n, r), **bf)
        wsb = fpq.fpq_qat_backward_workspace_bytes(m, n, k, r)
        self.ws = torch.empty(((wsb + 15) // 16 * 16,), dtype=torch.uint8, device=dev) if wsb else None
        u8 = dict(dtype=torch.uint8, device=dev)
        self.ws_g = torch.empty((fpq.fpq_qat_lora_grads_workspace_bytes(n, k, r),), **u8)
        self.dx_host = torch.empty((m, k), dtype=torch.bfloat16).pin_memory()
        self.da_host = torch.empty((r, k), dtype=torch.bfloat16).pin_memory()
        self.db_host = torch.empty((n, r), dtype=torch.bfloat16).pin_memory()
        self.flops = 2.0 * (2 * m * n * k + 2 * r * n * k)
        self.quant_bytes = 0.0          # no quantize kernel in this step
        self.launches = 4                # dA and dB: one fused pass over dW + the partial-sum reduction
        self.config = dict(self.CONFIG)

    def kernels(self):
        f, m, n, k, r, aor = self.f, self.m, self.n, self.k, self.r, self.aor
        return [
            ("gemm_bf16_dx", lambda: f.fpq_gemm_bf16_layout(self.dy, 0, self.w_fq, 1, m, k, n, 1.0, self.dx)),
            ("gemm_bf16_dw", lambda: f.fpq_gemm_bf16_layout(self.dy, 1, self.x_fq, 1, n, k, m, 1.0, self.dw)),
            ("lora_grads", lambda: f.fpq_qat_lora_grads(self.dw, self.a, self.b, n, k, r, aor, self.da, self.db,
                                                        self.ws_g)),
        ]

    def whole_step(self, side_stream):
        """The public call: dX on the library's second stream beside dW."""
        f = self.f
        f.fpq_qat_backward(self.dy, self.x_fq, self.w_fq, self.a, self.b, self.m, self.n, self.k, self.r, self.aor,
                           self.dx, self.dw, self.da, self.db, self.ws)

    def kernel_work(self):
        m, n, k, r = self.m, self.n, self.k, self.r
        return {"gemm_bf16_dx": ("TFLOP/s", 2.0 * m * n * k), "gemm_bf16_dw": ("TFLOP/s", 2.0 * m * n * k),
                # HBM-bound: dW, A, B read once, dA and dB written once
                "lora_grads": ("GB/s", 2.0 * (n * k + r * k + n * r) + 2.0 * (r * k + n * r))}

    def e2e_step(self, stream, side_stream):
        """dy from pinned host memory, the public fpq_qat_backward call, dx,
        dA and dB back to pinned host memory (dW_eff stays on the device)."""
        f = self.f
        self.dy.copy_(self.dy_host, non_blocking=True)
        f.fpq_qat_backward(self.dy, self.x_fq, self.w_fq, self.a, self.b, self.m, self.n, self.k, self.r, self.aor,
                           self.dx, self.dw, self.da, self.db, self.ws)
        self.dx_host.copy_(self.dx, non_blocking=True)
        self.da_host.copy_(self.da, non_blocking=True)
        self.db_host.copy_(self.db, non_blocking=True)
        return self.dy.numel() * 2, (self.dx.numel() + self.da.numel() + self.db.numel()) * 2


class Nvfp4Gemm(Step):
    """The fine-grained GEMM shape in NVFP4: both operands quantized on the
    GPU (packed E2M1, E4M3 scale per 16, fp32 tensor scale) and multiplied
    on the tensor cores (kind::mxf4nvf4, CTA pairs)."""
    name = "nvfp4_gemm"
    dominant = "gemm_nvfp4"
    CONFIG = {"workload": "nvfp4_gemm: A bf16 4096x7168 N(0,1) and B bf16 2048x7168 N(0,0.02) -> packed "
                          "E2M1 with E4M3 scale per 16 and fp32 tensor scale; C = gA gB A B^T fp32 "
                          "accumulate, bf16 out",
              "m": 4096, "n": 2048, "k": 7168, "l2": "flushed before every step (256 MiB write)"}
    dtype = "e2m1xe2m1->f32 (bf16 in/out)"
    tensor_ratio = 4.0         # dense fp4 / bf16, nominal 9 / 2.25
    side = ("quant_nvfp4_b",)          # B's quantizer runs beside A's
    join_before = "gemm_nvfp4"
    E2E_IN, E2E_OUT = ("a", "b"), ("c",)

    def __init__(self, fpq, dev, m=4096, n=2048, k=7168):
        self.f = fpq
        self.m, self.n, self.k = m, n, k
        wl = workloads.ds_fp8_gemm(m, n, k)
        self.a_host, self.b_host = wl["a"].pin_memory(), wl["b"].pin_memory()
        self.a, self.b = self.a_host.to(dev), self.b_host.to(dev)
        u8 = dict(dtype=torch.uint8, device=dev)
        self.qa, self.sa = torch.empty((m, k // 2), **u8), torch.empty((m, k // 16), **u8)
        self.qb, self.sb = torch.empty((n, k // 2), **u8), torch.empty((n, k // 16), **u8)
        self.ga = torch.empty((1,), dtype=torch.float32, device=dev)
        self.gb = torch.empty((1,), dtype=torch.float32, device=dev)
        wsb = (max(1, fpq.fpq_quantize_workspace_bytes(fpq.NVFP4, 1)) + 15) // 16 * 16
        self.wsa, self.wsb = torch.empty((wsb,), **u8), torch.empty((wsb,), **u8)
        self.c = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        self.c_host = torch.empty((m, n), dtype=torch.bfloat16).pin_memory()
        self.flops = 2.0 * m * n * k
        # algorithmic bytes: bf16 read once, codes and scales written once
        self.qa_bytes = m * k * (2 + 0.5 + 1 / 16) + 4
        self.qb_bytes = n * k * (2 + 0.5 + 1 / 16) + 4
        self.quant_bytes = self.qa_bytes + self.qb_bytes
        self.launches = 3      # two quantize kernels (each after a workspace memset) and the GEMM
        self.config = dict(self.CONFIG)

    def kernels(self):
        f = self.f
        return [
            ("quant_nvfp4_a", lambda: f.fpq_quantize_block(f.NVFP4, self.a, 1, self.m, self.k, self.qa, self.sa,
                                                           self.ga, self.wsa)),
            ("quant_nvfp4_b", lambda: f.fpq_quantize_block(f.NVFP4, self.b, 1, self.n, self.k, self.qb, self.sb,
                                                           self.gb, self.wsb)),
            ("gemm_nvfp4", lambda: f.fpq_scaled_gemm_nvfp4(self.qa, self.sa, self.ga, self.qb, self.sb, self.gb,
                                                           self.m, self.n, self.k, self.c, f.OUT_BF16)),
        ]

    def kernel_work(self):
        return {"quant_nvfp4_a": ("GB/s", self.qa_bytes), "quant_nvfp4_b": ("GB/s", self.qb_bytes),
                "gemm_nvfp4": ("TFLOP/s", self.flops)}

    def e2e_step(self, stream, side_stream):
        self.a.copy_(self.a_host, non_blocking=True)
        self.b.copy_(self.b_host, non_blocking=True)
        self.whole_step(side_stream)
        self.c_host.copy_(self.c, non_blocking=True)
        return self.a_host.numel() * 2 + self.b_host.numel() * 2, self.c.numel() * 2


class MoeDispatch(Step):
    """The FP8 MoE dispatch on one GPU: 16384 tokens x 7168 bf16, top-8 of 64
    experts; route (per-chunk histograms + scan), layout, and the fused
    kernel that quantizes each token row once to MXFP8 and writes it to the
    rows of its 8 experts in the expert-grouped buffer (the grouped GEMM's
    input).  On one GPU every destination is local."""
    name = "moe_dispatch"
    dominant = "moe_dispatch_mxfp8"
    CONFIG = {"workload": "moe_dispatch: X 16384x7168 bf16 N(0,1), top-8 of 64 experts (Gumbel-top-8 on "
                          "log((e+1)^-1.1)) -> MXFP8 rows grouped by expert, one GPU (all destinations "
                          "local)", "tokens": 16384, "hidden": 7168, "experts": 64, "topk": 8, "l2": "flushed before every step (256 MiB write)"}
    unit = "GB/s"
    dtype = "bf16 -> e4m3 + e8m0 (scatter)"

    def __init__(self, fpq, dev, tokens=16384, hidden=7168, experts=64, topk=8):
        self.f = fpq
        wl = workloads.moe_dispatch(tokens, experts, hidden, topk)
        self.x_host, self.ids_host = wl["x"][0].pin_memory(), wl["topk_ids"][0].pin_memory()
        self.x, self.ids = self.x_host.to(dev), self.ids_host.to(dev)
        self.t, self.h, self.e, self.k = tokens, hidden, experts, topk
        i32, i64, u8 = (dict(dtype=d, device=dev) for d in (torch.int32, torch.int64, torch.uint8))
        self.counts = torch.empty((experts,), **i32)
        wsb = fpq.fpq_moe_route_workspace_bytes(tokens, experts)
        self.ws = torch.empty(((wsb + 15) // 16 * 16,), **u8)
        self.row0 = torch.empty((experts,), **i64)
        self.offs = torch.empty((experts + 1,), **i32)
        rows = tokens * topk
        self.q, self.s = torch.empty((rows, hidden), **u8), torch.empty((rows, hidden // 32), **u8)
        self.qp = torch.tensor([self.q.data_ptr()], **i64)
        self.sp = torch.tensor([self.s.data_ptr()], **i64)
        self.cap = torch.tensor([rows], **i64)
        self.offs_host = torch.empty((experts + 1,), dtype=torch.int32).pin_memory()
        # algorithmic bytes: x read once, ids read twice (route, dispatch), codes + scales written once per pair
        self.dispatch_bytes = tokens * hidden * 2 + tokens * topk * 4 + rows * (hidden + hidden // 32)
        self.route_bytes = tokens * topk * 4
        self.bytes = self.dispatch_bytes + self.route_bytes
        self.quant_bytes = self.bytes
        self.launches = 4
        self.config = dict(self.CONFIG)

    @property
    def work(self):
        return self.bytes

    def kernels(self):
        f = self.f
        return [
            ("moe_route", lambda: f.fpq_moe_route(self.ids, self.t, self.k, self.e, self.counts, self.ws)),
            ("moe_layout", lambda: f.fpq_moe_dispatch_layout(self.counts, 1, self.e, 0, f.MOE_DIRECT, self.row0,
                                                             self.offs)),
            ("moe_dispatch_mxfp8", lambda: f.fpq_moe_dispatch_mxfp8(self.x, self.t, self.h, self.ids, self.k, self.e,
                                                                    self.ws, self.row0, 1, self.qp, self.sp,
                                                                    self.cap)),
        ]

    def kernel_work(self):
        return {"moe_route": ("GB/s", self.route_bytes), "moe_layout": ("GB/s", self.e * 4 * 2),
                "moe_dispatch_mxfp8": ("GB/s", self.dispatch_bytes)}

    def e2e_step(self, stream, side_stream):
        """Tokens and routing from pinned host memory in, the group offsets
        back to the host (the grouped rows stay on the device for the expert
        GEMM)."""
        self.x.copy_(self.x_host, non_blocking=True)
        self.ids.copy_(self.ids_host, non_blocking=True)
        self.whole_step(side_stream)
        self.offs_host.copy_(self.offs, non_blocking=True)
        return self.x_host.numel() * 2 + self.ids_host.numel() * 4, self.offs.numel() * 4


class Dequant(Step):
    """bf16 reconstruction of block-quantized tensors ("FP8 в DeepSeek V3",
    Практический смысл для инференс-инфраструктуры: FP8 weights converted
    back to BF16 where the hardware has no FP8 path): the 64-expert stacks
    of the prequant workload (gate, up [2048, 7168], down [7168, 2048]) from
    MXFP8 and from NVFP4, and the fine-grained operands (A 4096x7168 with
    1x128 fp32 scales, B 2048x7168 with 128x128 fp32 scales).  The codes
    and scales are made by the library once, outside the step; the step's
    work is the algorithmic bytes (codes and scales read, bf16 written)."""
    name = "dequant"
    CONFIG = {"workload": "dequant: 64 experts x {gate, up 2048x7168; down 7168x2048} from MXFP8 (1x32 E8M0) "
                          "and from NVFP4 (1x16 E4M3 + fp32 per matrix), A 4096x7168 from 1x128 fp32 scales, "
                          "B 2048x7168 from 128x128 fp32 scales -> bf16",
              "l2": "flushed before every step (256 MiB write)"}
    dominant = "dequant_mxfp8"
    unit = "GB/s"
    dtype = "e4m3 / e2m1 codes -> bf16 (fp32 scale arithmetic)"

    def __init__(self, fpq, dev, experts=64):
        self.f = fpq
        self.e = experts
        shapes = {"gate": (2048, 7168), "up": (2048, 7168), "down": (7168, 2048)}
        u8 = dict(dtype=torch.uint8, device=dev)
        self.mats = {}
        for i, (nm, (r, c)) in enumerate(shapes.items()):
            g = torch.Generator(device=dev)
            g.manual_seed(4000 + i)
            x = torch.empty((experts, r, c), dtype=torch.bfloat16, device=dev)
            for e in range(experts):
                x[e] = (torch.randn(r, c, generator=g, device=dev) * 0.02).to(torch.bfloat16)
            mq, ms = fpq.quantize(x, fpq.MXFP8)
            nq, ns, ng = fpq.quantize(x, fpq.NVFP4)
            self.mats[nm] = (r, c, mq, ms, nq, ns, ng, x)     # x is overwritten: it is the bf16 output
        wl = workloads.ds_fp8_gemm()
        a, b = wl["a"].to(dev), wl["b"].to(dev)
        self.aq, self.as_ = fpq.quantize(a, fpq.FP8_1x128)
        self.bq, self.bs = fpq.quantize(b, fpq.FP8_128x128)
        self.a_out, self.b_out = a, b
        elems = sum(experts * r * c for r, c, *_ in self.mats.values())
        self.mx_bytes = elems * (1 + 1 / 32 + 2)
        self.nv_bytes = elems * (0.5 + 1 / 16 + 2) + 4 * 3 * experts
        self.a_bytes = a.numel() * 3 + self.as_.numel() * 4
        self.b_bytes = b.numel() * 3 + self.bs.numel() * 4
        self.quant_bytes = self.mx_bytes + self.nv_bytes + self.a_bytes + self.b_bytes
        self.launches = 8
        self.config = dict(self.CONFIG)
        if experts != 64:
            self.config["workload"] = self.CONFIG["workload"].replace("64 experts", f"{experts} experts")

    @property
    def work(self) -> float:
        return self.quant_bytes

    def kernels(self):
        f = self.f

        def mx():
            for r, c, mq, ms, _, _, _, out in self.mats.values():
                f.fpq_dequantize(f.MXFP8, mq, ms, None, self.e, r, c, out)

        def nv():
            for r, c, _, _, nq, ns, ng, out in self.mats.values():
                f.fpq_dequantize(f.NVFP4, nq, ns, ng, self.e, r, c, out)

        return [("dequant_mxfp8", mx), ("dequant_nvfp4", nv),
                ("dequant_fp8_1x128", lambda: f.fpq_dequantize(f.FP8_1x128, self.aq, self.as_, None, 1, 4096, 7168,
                                                               self.a_out)),
                ("dequant_fp8_128x128", lambda: f.fpq_dequantize(f.FP8_128x128, self.bq, self.bs, None, 1, 2048,
                                                                 7168, self.b_out))]

    def kernel_work(self):
        return {"dequant_mxfp8": ("GB/s", self.mx_bytes), "dequant_nvfp4": ("GB/s", self.nv_bytes),
                "dequant_fp8_1x128": ("GB/s", self.a_bytes), "dequant_fp8_128x128": ("GB/s", self.b_bytes)}

    def e2e_step(self, stream, side_stream):
        """Codes and scales from pinned host memory in, every bf16 result
        back to pinned host memory, copies inside the timed region."""
        if not hasattr(self, "host"):
            self.host = []
            for r, c, mq, ms, nq, ns, ng, out in self.mats.values():
                self.host.append(([(t, t.cpu().pin_memory()) for t in (mq, ms, nq, ns, ng)],
                                  (out, torch.empty(out.shape, dtype=out.dtype).pin_memory())))
            self.host_ab = [(t, t.cpu().pin_memory()) for t in (self.aq, self.as_, self.bq, self.bs)]
            self.host_ab_out = [(t, torch.empty(t.shape, dtype=t.dtype).pin_memory()) for t in (self.a_out, self.b_out)]
        hb = db = 0
        for ins, _ in self.host:
            for d, h in ins:
                d.copy_(h, non_blocking=True)
                hb += h.numel() * h.element_size()
        for d, h in self.host_ab:
            d.copy_(h, non_blocking=True)
            hb += h.numel() * h.element_size()
        for _, fn in self.kernels():
            fn()
        for _, (d, h) in self.host:
            h.copy_(d, non_blocking=True)
            db += d.numel() * d.element_size()
        for d, h in self.host_ab_out:
            h.copy_(d, non_blocking=True)
            db += d.numel() * d.element_size()
        return hb, db


STEPS = {"ds_fp8_gemm": DsFp8Gemm, "moe_grouped": MoeGrouped, "qat_forward": QatForward,
         "moe_prequant": MoePrequant, "nvfp4_gemm": Nvfp4Gemm, "qat_backward": QatBackward,
         "moe_dispatch": MoeDispatch, "dequant": Dequant}


# ------------------------------------------------------------------ traffic from committed ncu summaries

def _source_hash(kernel: str) -> str | None:
    src = {"gemm_fp8_f32scale": "gemm_fp8_f32scale.cu", "gemm_grouped_mxfp8": "gemm_mxfp8.cu",
           "gemm_mxfp8": "gemm_mxfp8.cu", "quant_fp8_1x128": "quant_kernels.cu",
           "quant_mxfp8": "quant_kernels.cu", "lora_merge_fq": "merge_kernel.cu",
           "gemm_nvfp4": "gemm_nvfp4.cu", "gemm_bf16_dx": "gemm_bf16.cu",
           "moe_dispatch_mxfp8": "moe_dispatch.cu", "lora_grads": "lora_grads.cu",
           "quant_nvfp4": "quant_kernels.cu", "quant_fp8_128x128": "quant_kernels.cu",
           "dequant_mxfp8": "quant_kernels.cu"}.get(kernel)
    if not src:
        return None
    # the kernel's source file and every header of the library (a change in
    # a shared device helper changes the kernel too)
    csrc = os.path.join(ROOT, "mxfp8_block_scaled_warp_b200", "csrc")
    h = hashlib.sha256()
    for path in [os.path.join(csrc, src)] + sorted(glob.glob(os.path.join(csrc, "*.cuh")) +
                                                   glob.glob(os.path.join(csrc, "*.h"))):
        with open(path, "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def _traffic(kernel: str, workload: str):
    """dram read+write bytes per launch recorded in profiles/<kernel>__<workload>.md
    ('dram_bytes_per_launch: X' and 'source_sha256_16: H'); null when absent
    or when the kernel's source has changed since the capture."""
    p = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(p):
        return None
    text = open(p).read()
    b = re.search(r"dram_bytes_per_launch:\s*([0-9.eE+]+)", text)
    h = re.search(r"source_sha256_16:\s*([0-9a-f]+)", text)
    if not b or not h or h.group(1) != _source_hash(kernel):
        return None
    return float(b.group(1))


# ------------------------------------------------------------------ CPU baseline (oracle)
#
# A workload on the oracle is a list of phases; each phase is `total` units
# of one kind (quantized rows, 128-row strips, dispatched tokens, fp64 GEMM
# entries) with `work` of the line's unit per unit (flops, or bytes for the
# GB/s workloads).  A timed sample runs the same fraction f of every phase's
# units; each phase's units are split into contiguous ranges over the host
# threads (the oracle's C calls release the GIL, so the threads run in
# parallel).  The whole-step time is extrapolated per phase (its measured
# time x total / units run), and `value` = the step's work / that time.

class OraclePhase:
    def __init__(self, label: str, total: int, work: float, fn):
        self.label, self.total, self.work, self.fn = label, int(total), float(work), fn


def host_threads() -> int:
    try:
        return max(1, len(os.sched_getaffinity(0)))
    except AttributeError:
        return os.cpu_count() or 1


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_phases(phases, fraction: float, threads: int):
    """Run `fraction` of every phase's units (at least one unit each) on
    `threads` threads; returns [(units, seconds)] per phase."""
    from concurrent.futures import ThreadPoolExecutor
    out = []
    with ThreadPoolExecutor(threads) as ex:
        for ph in phases:
            n = int(max(1, min(ph.total, round(fraction * ph.total))))
            cuts = np.linspace(0, n, min(threads, n) + 1).astype(np.int64)
            t0 = time.perf_counter()
            list(ex.map(lambda i: ph.fn(int(cuts[i]), int(cuts[i + 1])), range(len(cuts) - 1)))
            out.append((n, time.perf_counter() - t0))
    return out


def extrapolate(phases, runs):
    """(seconds of the whole step, work of the whole step) from a sample."""
    step_s = sum(dt * ph.total / n for ph, (n, dt) in zip(phases, runs))
    return step_s, sum(ph.total * ph.work for ph in phases)


def _entries(fn, rows: int, cols: int):
    """fn(rr, cc) over entry indices [lo, hi) spread across a rows x cols
    sample of quantized operands (each entry costs the same)."""
    def run(lo, hi):
        i = np.arange(lo, hi, dtype=np.int64)
        return fn(i % rows, (i * 7) % cols)
    return run


def oracle_phases(workload: str, oracle):
    """(phases, unit, description) of a workload on the oracle, or None."""
    k = 7168
    if workload in ("ds_fp8_gemm", "nvfp4_gemm"):
        m, n = 4096, 2048
        wl = workloads.ds_fp8_gemm(m, n, k)
        a, b = workloads.as_u16(wl["a"]), workloads.as_u16(wl["b"])
        if workload == "ds_fp8_gemm":
            qa, sa = oracle.quant_fp8_1x128(a[:64])
            qb, sb = oracle.quant_fp8_128x128(b[:256])
            return [OraclePhase("1x128 quantize of A (rows)", m, 0.0, lambda lo, hi: oracle.quant_fp8_1x128(a[lo:hi])),
                    OraclePhase("128x128 quantize of B (128-row strips)", n // 128, 0.0,
                                lambda lo, hi: oracle.quant_fp8_128x128(b[128 * lo:128 * hi])),
                    OraclePhase("fp64 GEMM entries (K=7168)", m * n, 2.0 * k,
                                _entries(lambda r, c: oracle.gemm_entries(0, qa, sa, 1, qb, sb, r, c), 64, 256))], \
                "TFLOP/s", "4096x2048x7168 fine-grained FP8 step"
        qa, sa, ga = oracle.quant_nvfp4(a[:64])
        qb, sb, gb = oracle.quant_nvfp4(b[:256])
        return [OraclePhase("NVFP4 quantize of A (rows)", m, 0.0, lambda lo, hi: oracle.quant_nvfp4(a[lo:hi])),
                OraclePhase("NVFP4 quantize of B (rows)", n, 0.0, lambda lo, hi: oracle.quant_nvfp4(b[lo:hi])),
                OraclePhase("fp64 GEMM entries (K=7168)", m * n, 2.0 * k,
                            _entries(lambda r, c: oracle.gemm_entries(3, qa, sa, 3, qb, sb, r, c, ag=ga, bg=gb),
                                     64, 256))], \
            "TFLOP/s", "4096x2048x7168 NVFP4 step"
    if workload == "qat_forward":
        m, n = 8192, 2048
        wl = workloads.qat_forward()
        w, la, lb, x = (workloads.as_u16(wl[t]) for t in ("w", "lora_a", "lora_b", "x"))
        aor = wl["alpha_over_r"]
        qw, sw, _ = oracle.lora_merge_fakequant(w[:128], la, lb[:128], aor)
        qx, sx = oracle.quant_fp8_1x128(x[:64])
        return [OraclePhase("LoRA merge + 128x128 fake-quant of W (128-row strips)", n // 128, 0.0,
                            lambda lo, hi: oracle.lora_merge_fakequant(w[128 * lo:128 * hi], la,
                                                                       lb[128 * lo:128 * hi], aor)),
                OraclePhase("1x128 quantize of X (rows)", m, 0.0, lambda lo, hi: oracle.quant_fp8_1x128(x[lo:hi])),
                OraclePhase("fp64 GEMM entries (K=7168)", m * n, 2.0 * k,
                            _entries(lambda r, c: oracle.gemm_entries(0, qx, sx, 1, qw, sw, r, c), 64, 128))], \
            "TFLOP/s", "8192x2048x7168 QAT forward step"
    if workload == "qat_backward":
        m, n, r = 8192, 2048, 16
        phases = []
        for kk, total, what in ((2048, m * k + r * k, "dX and dA"), (8192, n * k, "dW_eff"), (7168, n * r, "dB")):
            p = workloads.as_u16(workloads.normal_bf16((64, kk), 1.0, seed=6000 + kk))
            q = workloads.as_u16(workloads.normal_bf16((64, kk), 0.02, seed=6001 + kk))
            phases.append(OraclePhase(f"fp64 bf16-product entries of {what} (K={kk})", total, 2.0 * kk,
                                      _entries(lambda rr, cc, p=p, q=q: oracle.gemm_bf16_entries(p, q, rr, cc),
                                               64, 64)))
        return phases, "TFLOP/s", "QAT backward step (dX, dW_eff, dA, dB)"
    if workload in ("moe_grouped", "moe_dispatch"):
        tokens, experts, topk, n = 16384, 64, 8, 2048
        wl = workloads.moe_dispatch(tokens=tokens)
        x, ids = workloads.as_u16(wl["x"][0]), wl["topk_ids"][0].numpy()
        per_tok = k * 2 + topk * 8 + topk * (k + k // 32)
        dispatch = OraclePhase("dispatch (route, MXFP8 quantize, placement) of tokens", tokens,
                               per_tok if workload == "moe_dispatch" else 0.0,
                               lambda lo, hi: oracle.moe_dispatch([x[lo:hi]], [ids[lo:hi]], experts))
        if workload == "moe_dispatch":
            return [dispatch], "GB/s", "16384-token top-8 FP8 dispatch"
        codes, scales, _ = oracle.moe_dispatch([x[:32]], [ids[:32]], experts)[0]
        rows = codes.shape[0]
        wq, ws = oracle.quant_mxfp8(np.stack([workloads.as_u16(workloads.normal_bf16((64, k), 0.02, seed=5100 + e))
                                              for e in range(2)]))
        off2 = np.array([0, rows // 2, rows], np.int64)
        return [dispatch,
                OraclePhase("fp64 grouped MXFP8 GEMM entries (K=7168)", tokens * topk * n, 2.0 * k,
                            _entries(lambda rr, cc: oracle.grouped_gemm_entries(2, codes, scales, wq, ws, off2, rr, cc),
                                     rows, 64))], \
            "TFLOP/s", "16384-token step (dispatch + grouped GEMM, 131072x2048x7168)"
    if workload in ("moe_prequant", "dequant"):
        x = workloads.as_u16(workloads.normal_bf16((2048, k), 0.02, 4000))
        rows_total = 64 * 3 * 2048            # gate, up [2048, 7168] and down [7168, 2048]: 7168-element rows

        def rows_of(lo, hi):
            return x[np.arange(lo, hi) % 2048]

        if workload == "moe_prequant":
            return [OraclePhase("MXFP8 quantize (7168-element rows)", rows_total, k * (3 + 1 / 32),
                                lambda lo, hi: oracle.quant_mxfp8(rows_of(lo, hi))),
                    OraclePhase("NVFP4 quantize (7168-element rows)", rows_total, k * (2.5 + 1 / 16),
                                lambda lo, hi: oracle.quant_nvfp4(rows_of(lo, hi)))], \
                "GB/s", "64-expert prequant step"
        mq, ms = oracle.quant_mxfp8(x[:256])
        nq, ns, ng = oracle.quant_nvfp4(x[:256])
        a = workloads.as_u16(workloads.ds_fp8_gemm()["a"][:256])
        aq, as_ = oracle.quant_fp8_1x128(a)
        bq, bs = oracle.quant_fp8_128x128(x[:256])
        return [OraclePhase("MXFP8 dequantize (7168-element rows)", rows_total, k * (1 + 1 / 32 + 2),
                            lambda lo, hi: oracle.dequant_mxfp8(mq[np.arange(lo, hi) % 256],
                                                                ms[np.arange(lo, hi) % 256])),
                OraclePhase("NVFP4 dequantize (7168-element rows)", rows_total, k * (0.5 + 1 / 16 + 2),
                            lambda lo, hi: oracle.dequant_nvfp4(nq[np.arange(lo, hi) % 256],
                                                                ns[np.arange(lo, hi) % 256], ng)),
                OraclePhase("1x128 dequantize of A (rows)", 4096, k * 3 + (k // 128) * 4,
                            lambda lo, hi: oracle.dequant_fp8_1x128(aq[np.arange(lo, hi) % 256],
                                                                    as_[np.arange(lo, hi) % 256])),
                OraclePhase("128x128 dequantize of B (128-row strips)", 16, 128 * k * 3 + (k // 128) * 4,
                            lambda lo, hi: [oracle.dequant_fp8_128x128(bq[:128], bs[:1]) for _ in range(lo, hi)])], \
            "GB/s", "dequantize step (64-expert MXFP8 and NVFP4 stacks, 1x128 A, 128x128 B)"
    return None


def cpu_baseline(workload: str, budget_s: float = 8.0, threads: int | None = None):
    """The oracle as it stands, timed on a bounded sample of the workload:
    once on one thread and once with the sample's units split over every
    host core (about `budget_s` seconds each); both extrapolated to the
    whole step in the workload's unit."""
    import oracle
    oracle.build()
    oracle.lib()
    spec = oracle_phases(workload, oracle)
    if spec is None:
        return None
    phases, unit, what = spec
    threads = threads or host_threads()
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    calib = run_phases(phases, 0.0, 1)                      # one unit of each phase
    full_1 = extrapolate(phases, calib)[0]
    f1 = budget_s / full_1
    one = run_phases(phases, f1, 1)
    one_s, work = extrapolate(phases, one)
    many = run_phases(phases, f1 * threads, threads)
    many_s, _ = extrapolate(phases, many)

    def sample(runs):
        return "; ".join(f"{n} of {ph.total} {ph.label}" for ph, (n, _) in zip(phases, runs))

    return {"value": work / many_s / scale, "unit": unit, "work": work, "cores": threads, "kind": "oracle",
            "cpu": cpu_model(),
            "sample": f"{sample(many)}; {sum(dt for _, dt in many):.1f} s on {threads} threads, extrapolated to the "
                      f"{what} ({many_s:.0f} s)",
            "one_core": {"value": work / one_s / scale, "unit": unit, "cores": 1,
                         "sample": f"{sample(one)}; {sum(dt for _, dt in one):.1f} s on one thread, extrapolated "
                                   f"to the {what} ({one_s:.0f} s)"}}


# ------------------------------------------------------------------ main

def run_reference(args, rank, world):
    """The reference arm: the CPU oracle as it stands, on every host core.
    Each step runs the same bounded sample of the workload (a fixed fraction
    of every phase's units, sized so that warm-up and timed steps end within
    about two minutes); `ms_per_step` is the measured time of a sampled step
    and `value` the workload's rate over the timed steps."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    oracle.lib()
    spec = oracle_phases(args.workload, oracle)
    if spec is None:
        print(json.dumps({"impl": "reference", "unavailable": f"no oracle timing defined for {args.workload}"}))
        return
    phases, unit, what = spec
    threads = host_threads()
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    per_step_s = args.ref_step_s or min(4.0, max(0.5, 120.0 / (args.steps + args.warmup)))
    full_1 = extrapolate(phases, run_phases(phases, 0.0, 1))[0]
    frac = per_step_s * threads / full_1
    for _ in range(args.warmup):
        run_phases(phases, frac, threads)
    runs, step_ms = [], []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        runs.append(run_phases(phases, frac, threads))
        step_ms.append((time.perf_counter() - t0) * 1e3)
    agg = [(sum(r[i][0] for r in runs), sum(r[i][1] for r in runs)) for i in range(len(phases))]
    step_s, work = extrapolate(phases, agg)
    v = work / step_s / scale
    sample = "; ".join(f"{n} of {ph.total} {ph.label}" for ph, (n, _) in zip(phases, runs[0]))
    line = {"impl": "reference", "metric": METRIC, "value": v, "unit": unit, "n_gpus": 1, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": statistics.mean(step_ms),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(STEPS[args.workload].CONFIG),
            "step": f"a fixed sample of the {what} per step ({sample}); value = the whole step's work over its "
                    f"time extrapolated per phase from the timed steps ({step_s:.0f} s per whole step)",
            "cpu_baseline": {"value": v, "unit": unit, "cores": threads, "kind": "oracle", "cpu": cpu_model(),
                             "sample": sample},
            "e2e": {"value": v, "unit": unit, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


# ------------------------------------------------------------------ replicas

def init_replicas(world: int, backend: str = "nccl", device=None):
    """One process per GPU, no data-path collective: the process group only
    carries the barriers around the timed region and the max over ranks.
    Returns the torch.distributed module, or None for a single process."""
    if world <= 1:
        return None
    import torch.distributed as dist
    from datetime import timedelta
    kw = {"device_id": device} if backend == "nccl" and device is not None else {}
    dist.init_process_group(backend, timeout=timedelta(seconds=120), **kw)
    return dist


def max_over_ranks(value: float, pg, device=None) -> float:
    """The slowest rank's time (every rank takes this collective in step)."""
    if pg is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_rank_step: float, steps: int, total_ms: float) -> float:
    """Weak scaling: every rank runs the same step on its own data, so the
    job's throughput is all ranks' work over the slowest rank's time."""
    return world * flops_per_rank_step * steps / (total_ms * 1e-3) / 1e12


def whole_job_rate(world: int, work_per_rank_step: float, steps: int, total_ms: float, unit: str) -> float:
    """whole_job_tflops for either unit: TFLOP/s (flops) or GB/s (bytes)."""
    scale = 1e12 if unit == "TFLOP/s" else 1e9
    return world * work_per_rank_step * steps / (total_ms * 1e-3) / scale


METRIC = "quantize GB/s vs HBM peak; block-scaled FP8 GEMM TFLOPS vs FP8 tensor peak"


def launch_note(step) -> str:
    fork = ""
    if step.side:
        fork = f" ({', '.join(step.side)} on a second stream beside the kernels before {step.join_before})"
    elif type(step).whole_step is not Step.whole_step:
        fork = f" ({' '.join((type(step).whole_step.__doc__ or '').split())})"
    return (f"CUDA graph of the step replayed per timed step{fork}; per-kernel times from a second graph with "
            f"events around each kernel, one after another")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="fpq", choices=["fpq", "reference"])
    ap.add_argument("--workload", default="moe_grouped", choices=sorted(STEPS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--ref-step-s", type=float, default=None,
                    help="reference arm: seconds of oracle work per sampled step (default: about two minutes "
                         "over warm-up and timed steps, 0.5 to 4 s per step)")
    ap.add_argument("--experts", type=int, default=None,
                    help="moe_prequant only: experts per projection (default 64; fewer for small profiler captures)")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        return run_reference(args, rank, world)

    import mxfp8_block_scaled_warp_b200 as fpq
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = init_replicas(world, "nccl", dev)

    if args.experts and args.workload not in ("moe_prequant", "dequant"):
        raise SystemExit("--experts applies to --workload moe_prequant and dequant only")
    step = STEPS[args.workload](fpq, dev, **({"experts": args.experts} if args.experts else {}))
    stream = torch.cuda.current_stream()
    flush = torch.empty(FLUSH_BYTES, dtype=torch.uint8, device=dev)
    kern = step.kernels()
    names = [n for n, _ in kern]

    side_stream = torch.cuda.Stream()

    def one_step(events=None):
        for i, (_, fn) in enumerate(kern):
            if events is not None:
                events[i][0].record()
            fn()
            if events is not None:
                events[i][1].record()

    for _ in range(args.warmup):
        flush.zero_()
        one_step()
    torch.cuda.synchronize()
    assert fpq.fpq_get_device_error() == 0

    # The step is captured as CUDA graphs and replayed, so that host-side
    # launch work never leaves the GPU idle inside the timed region.  Two
    # graphs of the same launches: `whole` records events only before the
    # first and after the last kernel, so consecutive kernels keep their
    # programmatic-dependent-launch overlap (the step time and the headline
    # value come from it; independent kernels may run on a second stream
    # there); `split` records events around every kernel, one after another
    # (the per-kernel times and the roofline come from it).  The L2 flush runs
    # outside the graphs before every replay; each replay's events are read
    # before the next replay overwrites them.
    def capture(events_per_kernel):
        ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)]
              for _ in (kern if events_per_kernel else [None])]
        g = torch.cuda.CUDAGraph()
        cap = torch.cuda.Stream()
        cap.wait_stream(stream)
        with torch.cuda.stream(cap):
            with torch.cuda.graph(g, stream=cap):
                if events_per_kernel:
                    one_step(ev)
                else:
                    ev[0][0].record()
                    step.whole_step(side_stream)
                    ev[0][1].record()
        stream.wait_stream(cap)
        return g, ev

    whole, ev_whole = capture(False)
    split, ev_split = capture(True)
    for _ in range(args.warmup):
        flush.zero_()
        whole.replay()
        flush.zero_()
        split.replay()
    torch.cuda.synchronize()
    assert fpq.fpq_get_device_error() == 0

    per_kernel = {n: [] for n in names}
    step_ms = []
    if pg:
        pg.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for s in range(args.steps):
            flush.zero_()
            whole.replay()
            ev_whole[0][1].synchronize()
            step_ms.append(ev_whole[0][0].elapsed_time(ev_whole[0][1]))
        torch.cuda.synchronize()
    if pg:
        pg.barrier()
    with ClockSampler(local) as clk_k:
        for s in range(args.steps):
            flush.zero_()
            split.replay()
            ev_split[-1][1].synchronize()
            for i, n in enumerate(names):
                per_kernel[n].append(ev_split[i][0].elapsed_time(ev_split[i][1]))
        torch.cuda.synchronize()
    status = fpq.fpq_get_device_error()
    if status != 0:
        raise SystemExit(f"device error word {status} after the timed steps")
    del whole, split
    total_ms = max_over_ranks(sum(step_ms), pg, dev)
    ms_per_step = total_ms / args.steps
    value = whole_job_rate(world, step.work, args.steps, total_ms, step.unit)

    peaks = _peaks()
    fp8_peak_burst = 2.0 * peaks["bf16_tflops"]
    # The per-kernel times come from steps replayed back to back.  When the
    # clock record of that loop shows the power cap (or the SM clock held
    # below its maximum), the kernels ran under sustained load and the tensor
    # peak is the measured sustained bf16 rate; otherwise the burst rate.
    ck = clk_k.summary()
    sustained = bool(peaks.get("bf16_tflops_sustained")) and (
        "sw_power_cap" in ck["reasons"] or
        (ck["sm_mhz"] is not None and ck["sm_max_mhz"] and ck["sm_mhz"] < 0.97 * ck["sm_max_mhz"]))
    bf16_peak = peaks["bf16_tflops_sustained"] if sustained else peaks["bf16_tflops"]
    tensor_peak = step.tensor_ratio * bf16_peak
    tensor_peak_burst = step.tensor_ratio * peaks["bf16_tflops"]
    kernels_out = {}
    for n in names:
        unit, work = step.kernel_work()[n]
        ms = statistics.mean(per_kernel[n])
        ach = work / (ms * 1e-3) / (1e9 if unit == "GB/s" else 1e12)
        pk = peaks["hbm_gbs"] if unit == "GB/s" else tensor_peak
        kernels_out[n] = {"ms": ms, "achieved": ach, "unit": unit, "frac_of_peak": ach / pk}
    dom = kernels_out[step.dominant]
    traffic = _traffic(step.dominant, step.name)
    if dom["unit"] == "GB/s":
        roofline = {"kernel": step.dominant, "bound": "hbm", "achieved": dom["achieved"], "peak": peaks["hbm_gbs"],
                    "unit": "GB/s", "frac": dom["achieved"] / peaks["hbm_gbs"], "traffic": traffic,
                    "peak_note": f"{peaks['source']} HBM copy bandwidth"}
    else:
        kind = {4.0: "fp4", 2.0: "fp8", 1.0: "bf16"}[step.tensor_ratio]
        which = "sustained" if sustained else "burst"
        roofline = {"kernel": step.dominant, "bound": "tensor", "achieved": dom["achieved"], "peak": tensor_peak,
                    "unit": "TFLOP/s", "frac": dom["achieved"] / tensor_peak, "traffic": traffic,
                    "peak_kind": which, "frac_of_burst": dom["achieved"] / tensor_peak_burst,
                    "peak_note": f"{kind} = {step.tensor_ratio:g} x {peaks['source']} cuBLAS bf16 {which} "
                                 f"({bf16_peak} TFLOP/s; nominal dense ratio); {which} because the kernel-timing "
                                 f"loop's clock record {'shows' if sustained else 'does not show'} the power cap"}
    quant_ms = sum(statistics.mean(per_kernel[n]) for n in names if not n.startswith("gemm"))
    quant_gbs = step.quant_bytes / (quant_ms * 1e-3) / 1e9 if quant_ms > 0 else None

    # end to end: host buffers through the public API, copies inside the timed region
    e2e = None
    if hasattr(step, "e2e_step"):
        for _ in range(2):
            step.e2e_step(stream, side_stream)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        reps = max(3, min(args.steps, 20))
        e0.record(stream)
        for _ in range(reps):
            hb, db = step.e2e_step(stream, side_stream)
        e1.record(stream)
        e1.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1) / reps, pg, dev)
        e2e = {"value": whole_job_rate(world, step.work, 1, e2e_ms, step.unit), "unit": step.unit, "h2d_bytes_per_step": hb,
               "d2h_bytes_per_step": db, "ms_per_step": e2e_ms, "loop": "one step after another"}
        if step.E2E_IN:
            step.e2e_pipelined(2, side_stream)
            p_ms, hb, db = step.e2e_pipelined(reps, side_stream)
            p_ms = max_over_ranks(p_ms, pg, dev)
            e2e = {"value": whole_job_rate(world, step.work, 1, p_ms, step.unit), "unit": step.unit,
                   "h2d_bytes_per_step": hb, "d2h_bytes_per_step": db, "ms_per_step": p_ms,
                   "loop": "serving loop: each step's upload and readback on copy streams, two slots of inputs "
                           "and outputs, overlapping the neighbouring steps' kernels",
                   "one_after_another": {"value": e2e["value"], "ms_per_step": e2e_ms}}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(step.name)

    line = {"metric": METRIC, "value": value, "unit": step.unit, "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": step.dtype, "data": "synthetic",
            "config": dict(step.CONFIG), "workload_detail": step.config, "launch": launch_note(step),
            "quantize_gbs": quant_gbs,
            "quantize_frac_of_hbm": quant_gbs / peaks["hbm_gbs"] if quant_gbs is not None else None,
            "kernels": kernels_out, "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": step.launches * args.steps, "clocks": clk.summary(), "clocks_kernel_timing": ck,
            "peaks": {"hbm_gbs": peaks["hbm_gbs"], "fp8_tflops": fp8_peak_burst, "tensor_tflops": tensor_peak,
                      "source": peaks["source"]}}
    if rank == 0:
        print(json.dumps(line))
    if pg:
        pg.destroy_process_group()


if __name__ == "__main__":
    main()
