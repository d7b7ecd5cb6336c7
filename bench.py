#!/usr/bin/env python
"""Benchmark of the block-scaled FP4 path on B200.

One step = one pass of the whole path over one synthetic workload.  The
default workload is the whole weight set of a 7B-class decoder (32 layers x
(4 x 4096x4096 + 3 x 4096x14336) bf16, 224 matrices, 7.78e9 elements,
15.6 GB), each matrix with its own tensor amax and global scale:
  grouped tensor amax -> grouped NVFP4 quantise + pack -> grouped MXFP4
  quantise + pack -> grouped NVFP4 and MXFP4 dequantise (bf16)
(5 kernel launches).  The single-tensor workloads (--workload) run
  tensor amax -> NVFP4 quantise + pack -> MXFP4 quantise + pack ->
  NVFP4 dequantise (bf16) -> MXFP4 dequantise (bf16) -> NVFP4 scale search
(6 launches; the amax is shared by the NVFP4 quantiser and the search).
`value` is elements per second over the whole job, timed on the device
with CUDA events around each step, L2 flushed (512 MiB write, 256 MiB read)
between steps, max over ranks; nothing is recorded between the launches of
a step (an event there would serialise them).  Per-kernel times come from a
second pass with an event after every launch.  `e2e` times the same step
through the same C-ABI calls starting from pinned host memory: host->device
copy of x, the step, device->host copy of every quantised artefact and the
status word.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
    python bench.py --impl reference ...   # the CPU oracle on host cores

Multi-GPU (torchrun), two modes:
  --shard replicas (default)  every rank quantises its own tensor or weight
      set (independent problems, seeds offset by rank): weak scaling, no
      collective on the data path; one max all-reduce of the timings.
  --shard rows  one tensor of a single-tensor workload split by rows across
      the ranks; the step's only exchange is one max all-reduce of the
      4-byte tensor amax between the per-rank amax and the NVFP4
      quantiser / search: strong scaling.
"""
from __future__ import annotations

import argparse
import ctypes
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = "FP4 quantize elements/s and achieved HBM GB/s (fraction of B200 peak), 1 GPU"
WORKLOADS = {
    "weight-4096x4096-bf16": workloads.WEIGHT_4K,
    "act-8192x14336-bf16": workloads.ACT_8K,
    "search-4096x14336-bf16": workloads.SEARCH_4K,
    "tiny-f32-256x1024": workloads.TINY_F32,
    "model-7b-weights-bf16": workloads.MODEL_WEIGHTS,
    "columns-4096x14336-bf16": workloads.COLUMNS_4K,
    "ragged-8192x14335-bf16": workloads.RAGGED_8K,
    "variants-8192x14336-bf16": workloads.VARIANTS_8K,
    "gemm-8192x4096x14336-nvfp4": workloads.GEMM_ACT,
}
GEMM_WORKLOAD = "gemm-8192x4096x14336-nvfp4"
LAYOUT_WORKLOADS = {"columns-4096x14336-bf16": "columns", "ragged-8192x14335-bf16": "padded",
                    "variants-8192x14336-bf16": "variants"}
MODEL_WEIGHTS = "model-7b-weights-bf16"  # the whole weight set, grouped calls
DEFAULT_WORKLOAD = MODEL_WEIGHTS
KERNEL_SOURCES = ["block_scaled_fp4_reduce_b200/csrc/fp4_kernels.cuh",
                  "block_scaled_fp4_reduce_b200/csrc/fp4_codec.cuh",
                  "block_scaled_fp4_reduce_b200/csrc/fp4_grouped.cuh"]
LAYOUT_SOURCES = ["block_scaled_fp4_reduce_b200/csrc/fp4_layouts.cuh"]
GEMM_SOURCES = ["block_scaled_fp4_reduce_b200/csrc/fp4_gemm.cuh", "block_scaled_fp4_reduce_b200/csrc/fp4_gemm.cu"]
OPS = ["amax", "nvfp4_quantize", "mxfp4_quantize", "nvfp4_dequantize", "mxfp4_dequantize", "scale_search"]


def peaks() -> dict:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": float(d["hbm_gbs"]), "sm_max_mhz": float(d.get("sm_max_mhz", 1965.0)),
                "bf16_tflops": float(d.get("bf16_tflops", 1590.0)), "source": "measured"}
    return {"hbm_gbs": 6650.0, "sm_max_mhz": 1965.0, "bf16_tflops": 1590.0, "source": "fallback"}


def kernel_source_hash(extra: tuple = ()) -> str:
    """Hash of the kernel sources a traffic capture was taken from (the
    layout and GEMM workloads' kernels also live in the sources
    traffic_sources names)."""
    h = hashlib.sha256()
    for rel in list(KERNEL_SOURCES) + list(extra):
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def algorithmic_bytes(w: workloads.Workload) -> dict:
    """Bytes each kernel must move per launch (read + write), by definition:
    x once per pass, packed codes 1/2 byte per element, one scale byte per
    block, dequantised bf16 output 2 bytes per element (the grouped weight
    set: the same per element over all its matrices)."""
    n, e = w.numel, (2 if w.dtype == torch.bfloat16 else 4)
    return {
        "amax": n * e,
        "nvfp4_quantize": n * e + n // 2 + n // 16,
        "mxfp4_quantize": n * e + n // 2 + n // 32,
        "nvfp4_dequantize": n // 2 + n // 16 + 2 * n,
        "mxfp4_dequantize": n // 2 + n // 32 + 2 * n,
        "scale_search": n * e + n // 2 + n // 16,
        "scales_to_mma": 2 * (n // 16),
    }


# ---------------------------------------------------------------- clocks --

class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons (every 100 ms,
    read-only queries).  Sampling starts before the timed region and waits
    for the first sample, so that even a short region is covered; `stop`
    keeps the samples whose timestamps fall inside the region (all of them
    when none does, and says so)."""
    FIELDS = ["timestamp", "clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.active",
              "clocks_event_reasons.hw_slowdown", "clocks_event_reasons.hw_thermal_slowdown",
              "clocks_event_reasons.sw_thermal_slowdown", "clocks_event_reasons.sw_power_cap"]
    REASONS = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]

    def __init__(self, device: int):
        self.proc = None
        self.out = None
        self.t0 = self.t1 = None
        try:
            uuid = str(torch.cuda.get_device_properties(device).uuid)
            self.target = uuid if uuid.startswith("GPU-") else f"GPU-{uuid}"
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
            self.target = vis.split(",")[device] if vis else str(device)

    def start(self, wait_s: float = 5.0):
        try:
            self.out = open(os.path.join("/tmp", f"clocks_{os.getpid()}.csv"), "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.target, f"--query-gpu={','.join(self.FIELDS)}",
                 "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.out, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
            return
        t_end = time.time() + wait_s  # until the first sample is written
        while time.time() < t_end and self.proc.poll() is None:
            if os.path.getsize(self.out.name) > 0:
                break
            time.sleep(0.02)

    def mark(self, begin: bool):
        """Wall-clock bounds of the timed region."""
        if begin:
            self.t0 = time.time()
        else:
            self.t1 = time.time()

    @staticmethod
    def _stamp(s: str):
        try:
            return datetime.datetime.strptime(s, "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        time.sleep(0.25)  # one more sample after the region
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.out.name) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == len(self.FIELDS):
                    rows.append(parts)
        os.unlink(self.out.name)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        window = "timed region"
        if self.t0 is not None and self.t1 is not None:
            inside = [r for r in rows if (t := self._stamp(r[0])) is not None and self.t0 - 0.05 <= t <= self.t1 + 0.15]
            if inside:
                rows = inside
            else:
                window = "sampler run (no sample inside the timed region)"

        def num(s):
            try:
                return float(s)
            except ValueError:
                return None
        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        mx = [num(r[2]) for r in rows if num(r[2]) is not None]
        reasons = sorted({self.REASONS[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": reasons, "samples": len(rows), "window": window}


# -------------------------------------------------------------- the step --

class Path:
    """Device buffers and pre-bound C-ABI calls of one step."""

    def __init__(self, x: torch.Tensor):
        import block_scaled_fp4_reduce_b200 as fp4
        self.fp4 = fp4
        L = fp4.lib()
        dev = x.device
        R, C = x.shape
        self.x = x
        self.n = x.numel()
        u8 = torch.uint8
        self.amax = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws = fp4.workspace_for(x)
        self.status = fp4.new_status(dev)
        self.nv_p = torch.empty((R, C // 2), dtype=u8, device=dev)
        self.nv_s = torch.empty((R, C // 16), dtype=u8, device=dev)
        self.nv_g = torch.empty(1, dtype=torch.float32, device=dev)
        self.mx_p = torch.empty((R, C // 2), dtype=u8, device=dev)
        self.mx_s = torch.empty((R, C // 32), dtype=u8, device=dev)
        self.y_nv = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
        self.y_mx = torch.empty((R, C), dtype=torch.bfloat16, device=dev)
        self.ss_p = torch.empty((R, C // 2), dtype=u8, device=dev)
        self.ss_s = torch.empty((R, C // 16), dtype=u8, device=dev)
        self.ss_g = torch.empty(1, dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream().cuda_stream
        dt = fp4._dtype_code(x)
        P = lambda t: t.data_ptr()  # noqa: E731
        self.calls = [
            (L.fp4_tensor_amax, (P(x), dt, self.n, P(self.amax), P(self.ws), self.ws.numel(), P(self.status), st)),
            (L.fp4_nvfp4_quantize_with_amax, (P(x), dt, R, C, P(self.amax), P(self.nv_p), P(self.nv_s),
                                              P(self.nv_g), P(self.status), st)),
            (L.fp4_mxfp4_quantize, (P(x), dt, R, C, P(self.mx_p), P(self.mx_s), P(self.status), st)),
            (L.fp4_dequantize, (fp4.NVFP4, P(self.nv_p), P(self.nv_s), P(self.nv_g), R, C, P(self.y_nv),
                                fp4.BF16, st)),
            (L.fp4_dequantize, (fp4.MXFP4, P(self.mx_p), P(self.mx_s), None, R, C, P(self.y_mx), fp4.BF16, st)),
            (L.fp4_scale_search_with_amax, (P(x), dt, R, C, P(self.amax), P(self.ss_p), P(self.ss_s),
                                            P(self.ss_g), None, P(self.status), st)),
        ]
        self.results = [self.nv_p, self.nv_s, self.nv_g, self.mx_p, self.mx_s, self.ss_p, self.ss_s,
                        self.status]

    OPS = OPS
    LAUNCHES = 6  # one kernel per entry point (the amax folds in its last CTA)

    def twin(self, x2: torch.Tensor) -> "Path":
        """The same step on another input buffer with its own outputs (the
        second half of the double-buffered end-to-end pipeline)."""
        return Path(x2)

    def step(self, events=None):
        for i, (fn, args) in enumerate(self.calls):
            st = fn(*args)
            if st != 0:
                raise self.fp4.FP4Error(st, fn.__name__)
            if events is not None:
                events[i + 1].record()

    def check_status(self):
        st = int(self.status.item())
        if st:
            raise self.fp4.FP4Error(st, "bench step")


def shard_rows(rows: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) of rank `rank` when `rows` rows are split into `world`
    contiguous shards, the first rows % world of them one row longer."""
    base, extra = divmod(rows, world)
    r0 = rank * base + min(rank, extra)
    return r0, r0 + base + (1 if rank < extra else 0)


def sharded_step(local_amax, all_reduce_max, rest):
    """One row-sharded step: this rank's tensor amax, the max all-reduce
    that makes it the whole tensor's A (the step's only exchange: the blocks
    themselves are independent), then the rest of the step with that A.
    The callables act on the amax in place; `rest` returns the step's
    result."""
    a = local_amax()
    all_reduce_max(a)
    return rest(a)


class ShardedPath(Path):
    """The single-tensor step on this rank's rows of a tensor split across
    ranks: fp4_tensor_amax of the shard -> all-reduce(MAX) of the 4-byte A
    over the ranks (NCCL) -> the NVFP4 quantiser and the search with that A
    (fp4_*_with_amax), the MXFP4 quantiser and both dequantisers as on one
    GPU.  Each rank reads only its own memory."""
    OPS = ["amax", "amax_allreduce"] + OPS[1:]

    def __init__(self, x: torch.Tensor):
        super().__init__(x)
        import torch.distributed as dist
        self.dist = dist

    def twin(self, x2: torch.Tensor) -> "ShardedPath":
        return ShardedPath(x2)

    def step(self, events=None):
        def call(i):
            fn, args = self.calls[i]
            st = fn(*args)
            if st != 0:
                raise self.fp4.FP4Error(st, fn.__name__)

        def local_amax():
            call(0)
            if events is not None:
                events[1].record()
            return self.amax

        def all_reduce_max(a):
            self.dist.all_reduce(a, op=self.dist.ReduceOp.MAX)
            if events is not None:
                events[2].record()

        def rest(_a):
            for i in range(1, len(self.calls)):
                call(i)
                if events is not None:
                    events[i + 2].record()

        sharded_step(local_amax, all_reduce_max, rest)


def layer_spans(sizes: list[int], per: int) -> list[tuple[int, int, int, int]]:
    """The weight set's layers for the layer-streamed end-to-end run: per
    layer (first item, items, first element, end element) of consecutive
    groups of `per` items (the last group may be short), items laid out one
    after another in element order."""
    spans, e0 = [], 0
    for li in range(0, len(sizes), per):
        e1 = e0 + sum(sizes[li:li + per])
        spans.append((li, min(per, len(sizes) - li), e0, e1))
        e0 = e1
    return spans


class GroupedPath:
    """The whole 7B-class weight set (32 layers x 4 x 4096^2 + 3 x 4096x14336
    bf16 matrices, each generated from its own seed) in one flat device
    buffer; one step = grouped amax, grouped NVFP4 quantise (per-matrix g),
    grouped MXFP4 quantise, grouped NVFP4 and MXFP4 dequantise to bf16: five
    entry points, one kernel each (plus the clear of the amax words)."""
    OPS = ["amax", "nvfp4_quantize", "mxfp4_quantize", "nvfp4_dequantize", "mxfp4_dequantize"]
    LAUNCHES = 5

    def __init__(self, device, rank: int = 0, layers: int = workloads.MODEL_LAYERS):
        import block_scaled_fp4_reduce_b200 as fp4
        self.fp4 = fp4
        L = fp4.lib()
        self.ws_list = [workloads.model_matrix(l, i) for l in range(layers)
                        for i in range(len(workloads.MODEL_MATRICES))]
        if rank:
            self.ws_list = [workloads.for_rank(w, rank) for w in self.ws_list]
        sizes = [w.numel for w in self.ws_list]
        self.n = sum(sizes)
        u8, bf = torch.uint8, torch.bfloat16
        self.x = torch.empty(self.n, dtype=bf, device=device)
        off, self.xs = 0, []
        for w, m in zip(self.ws_list, sizes):
            v = self.x[off:off + m].view(w.rows, w.cols)
            v.copy_(workloads.generate(w, device=device))
            self.xs.append(v)
            off += m
        n = self.n
        self.nv_p, self.nv_s = torch.empty(n // 2, dtype=u8, device=device), torch.empty(n // 16, dtype=u8, device=device)
        self.mx_p, self.mx_s = torch.empty(n // 2, dtype=u8, device=device), torch.empty(n // 32, dtype=u8, device=device)
        self.nv_g = torch.empty(len(sizes), dtype=torch.float32, device=device)
        self.y_nv = torch.empty(n, dtype=bf, device=device)
        self.y_mx = torch.empty(n, dtype=bf, device=device)
        self.ws = torch.empty(L.fp4_grouped_workspace_bytes(len(sizes)), dtype=u8, device=device)
        self.status = fp4.new_status(device)
        k = len(sizes)
        self.q_nv = (fp4.QuantItem * k)()
        self.q_mx = (fp4.QuantItem * k)()
        self.d_nv = (fp4.DequantItem * k)()
        self.d_mx = (fp4.DequantItem * k)()
        off = 0
        for j, (w, m) in enumerate(zip(self.ws_list, sizes)):
            P = lambda t, o: t.data_ptr() + o * t.element_size()  # noqa: E731
            self.q_nv[j] = fp4.QuantItem(P(self.x, off), w.rows, w.cols, P(self.nv_p, off // 2),
                                         P(self.nv_s, off // 16), P(self.nv_g, j))
            self.q_mx[j] = fp4.QuantItem(P(self.x, off), w.rows, w.cols, P(self.mx_p, off // 2),
                                         P(self.mx_s, off // 32), None)
            self.d_nv[j] = fp4.DequantItem(P(self.nv_p, off // 2), P(self.nv_s, off // 16), P(self.nv_g, j),
                                           P(self.y_nv, off), w.rows, w.cols)
            self.d_mx[j] = fp4.DequantItem(P(self.mx_p, off // 2), P(self.mx_s, off // 32), None,
                                           P(self.y_mx, off), w.rows, w.cols)
            off += m
        st = torch.cuda.current_stream().cuda_stream
        cp = lambda a: ctypes.cast(a, ctypes.c_void_p)  # noqa: E731
        ws, stp = self.ws.data_ptr(), self.status.data_ptr()
        self.calls = [
            (L.fp4_tensor_amax_grouped, (cp(self.q_nv), k, fp4.BF16, ws, self.ws.numel(), stp, st)),
            (L.fp4_nvfp4_quantize_grouped_with_amax, (cp(self.q_nv), k, fp4.BF16, ws, stp, st)),
            (L.fp4_mxfp4_quantize_grouped, (cp(self.q_mx), k, fp4.BF16, stp, st)),
            (L.fp4_dequantize_grouped, (fp4.NVFP4, cp(self.d_nv), k, fp4.BF16, st)),
            (L.fp4_dequantize_grouped, (fp4.MXFP4, cp(self.d_mx), k, fp4.BF16, st)),
        ]
        self.results = [self.nv_p, self.nv_s, self.nv_g, self.mx_p, self.mx_s, self.status]
        # The same five calls per layer (the layer's seven matrices), for the
        # end-to-end run that streams the set layer by layer: the elements
        # [e0, e1) of x that the layer holds, and its calls.
        self.layers = []
        for li, n_l, e0, e1 in layer_spans(sizes, len(workloads.MODEL_MATRICES)):
            sl = lambda a, j=li: ctypes.c_void_p(ctypes.addressof(a) + j * ctypes.sizeof(a._type_))  # noqa: E731
            calls = [
                (L.fp4_tensor_amax_grouped, (sl(self.q_nv), n_l, fp4.BF16, ws, self.ws.numel(), stp, st)),
                (L.fp4_nvfp4_quantize_grouped_with_amax, (sl(self.q_nv), n_l, fp4.BF16, ws, stp, st)),
                (L.fp4_mxfp4_quantize_grouped, (sl(self.q_mx), n_l, fp4.BF16, stp, st)),
                (L.fp4_dequantize_grouped, (fp4.NVFP4, sl(self.d_nv), n_l, fp4.BF16, st)),
                (L.fp4_dequantize_grouped, (fp4.MXFP4, sl(self.d_mx), n_l, fp4.BF16, st)),
            ]
            self.layers.append((e0, e1, calls))

    step = Path.step
    check_status = Path.check_status

    def layer_outputs(self, e0: int, e1: int):
        """(device tensor, slice) of every per-element result of elements
        [e0, e1): the NVFP4 and MXFP4 packed codes and scale bytes."""
        return [(self.nv_p, slice(e0 // 2, e1 // 2)), (self.nv_s, slice(e0 // 16, e1 // 16)),
                (self.mx_p, slice(e0 // 2, e1 // 2)), (self.mx_s, slice(e0 // 32, e1 // 32))]


class LayoutPath:
    """The other block layouts and scale rules on one tensor x [R, K]:
    "variants" = amax, NVFP4 four over six (it runs its own amax: two
    launches), MXFP4 with the ceil scale rule, dequantisation of both to
    bf16; "columns" = amax,
    column-wise NVFP4 quantise (Q(W^T), g from that amax), column-wise MXFP4
    quantise, dequantisation of both padded layouts of the [K, R] transpose
    to bf16; "padded" = amax, NVFP4 (from that amax) and MXFP4 quantise of
    rows padded to whole blocks, dequantisation of both back to the logical
    [R, K] bf16."""
    OPS = ["amax", "nvfp4_quantize", "mxfp4_quantize", "nvfp4_dequantize", "mxfp4_dequantize"]
    LAUNCHES = 5

    def twin(self, x2: torch.Tensor) -> "LayoutPath":
        return LayoutPath(x2, self.kind)

    def __init__(self, x: torch.Tensor, kind: str):
        import block_scaled_fp4_reduce_b200 as fp4
        self.fp4 = fp4
        L = fp4.lib()
        dev = x.device
        R, K = x.shape
        self.x, self.n, self.kind = x, x.numel(), kind
        u8 = torch.uint8
        if kind == "columns":  # outputs describe the [K, R] transpose
            OR, OC = K, R
        else:
            OR, OC = R, K
        pad = lambda c, gsz: -(-c // gsz) * gsz  # noqa: E731
        self.amax = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws = fp4.workspace_for(x)
        self.status = fp4.new_status(dev)
        self.nv_p = torch.empty((OR, pad(OC, 16) // 2), dtype=u8, device=dev)
        self.nv_s = torch.empty((OR, pad(OC, 16) // 16), dtype=u8, device=dev)
        self.nv_g = torch.empty(1, dtype=torch.float32, device=dev)
        self.mx_p = torch.empty((OR, pad(OC, 32) // 2), dtype=u8, device=dev)
        self.mx_s = torch.empty((OR, pad(OC, 32) // 32), dtype=u8, device=dev)
        self.y_nv = torch.empty((OR, OC), dtype=torch.bfloat16, device=dev)
        self.y_mx = torch.empty((OR, OC), dtype=torch.bfloat16, device=dev)
        st = torch.cuda.current_stream().cuda_stream
        dt = fp4._dtype_code(x)
        P = lambda t: t.data_ptr()  # noqa: E731
        ws_bytes = self.ws.numel()
        if kind == "variants":  # four over six (its own amax inside) and the MXFP4 ceil rule
            nv_call = (L.fp4_nvfp4_quantize_four_over_six, (P(x), dt, R, K, P(self.nv_p), P(self.nv_s), P(self.nv_g),
                                                           None, P(self.ws), ws_bytes, P(self.status), st))
            mx_call = (L.fp4_mxfp4_quantize_ceil, (P(x), dt, R, K, P(self.mx_p), P(self.mx_s), P(self.status), st))
        else:
            # the NV call takes the step's amax (one amax pass per step, as on the row path)
            nvq = (L.fp4_nvfp4_quantize_columns_with_amax if kind == "columns"
                   else L.fp4_nvfp4_quantize_padded_with_amax)
            mxq = L.fp4_mxfp4_quantize_columns if kind == "columns" else L.fp4_mxfp4_quantize_padded
            nv_call = (nvq, (P(x), dt, R, K, P(self.amax), P(self.nv_p), P(self.nv_s), P(self.nv_g),
                             P(self.status), st))
            mx_call = (mxq, (P(x), dt, R, K, fp4.MX_FLOOR, P(self.mx_p), P(self.mx_s), P(self.status), st))
        self.calls = [
            (L.fp4_tensor_amax, (P(x), dt, self.n, P(self.amax), P(self.ws), ws_bytes, P(self.status), st)),
            nv_call,
            mx_call,
            (L.fp4_dequantize_padded, (fp4.NVFP4, P(self.nv_p), P(self.nv_s), P(self.nv_g), OR, OC,
                                       P(self.y_nv), fp4.BF16, st)),
            (L.fp4_dequantize_padded, (fp4.MXFP4, P(self.mx_p), P(self.mx_s), None, OR, OC, P(self.y_mx),
                                       fp4.BF16, st)),
        ]
        self.results = [self.nv_p, self.nv_s, self.nv_g, self.mx_p, self.mx_s, self.status]

        if kind == "variants":
            self.LAUNCHES = 6

    step = Path.step
    check_status = Path.check_status


class GemmPath:
    """The consumer: per step the activation x [M, K] is quantised (tensor
    amax, NVFP4 quantise, scales to the MMA layout) and multiplied on the
    tensor cores by the weight W [N, K], quantised once before timing:
    D [M, N] fp32 = g_x g_w x_hat W_hat^T."""
    OPS = ["amax", "nvfp4_quantize", "scales_to_mma", "nvfp4_gemm"]
    LAUNCHES = 4

    def __init__(self, x: torch.Tensor, w: torch.Tensor = None, shared: "GemmPath" = None):
        import block_scaled_fp4_reduce_b200 as fp4
        self.fp4 = fp4
        L = fp4.lib()
        dev = x.device
        M, K = x.shape
        u8 = torch.uint8
        if shared is None:
            qw = fp4.nvfp4_quantize(w)
            self.w_sf = fp4.scales_to_mma(qw.scales)
            torch.cuda.synchronize()
            qw.check()
        else:  # the quantised weight of another path, read-only
            qw, self.w_sf = shared.qw, shared.w_sf
        self.qw = qw
        N = qw.rows
        self.x, self.n, self.M, self.N, self.K = x, x.numel(), M, N, K
        self.amax = torch.empty(1, dtype=torch.float32, device=dev)
        self.ws = fp4.workspace_for(x)
        self.status = fp4.new_status(dev)
        self.p = torch.empty((M, K // 2), dtype=u8, device=dev)
        self.s = torch.empty((M, K // 16), dtype=u8, device=dev)
        self.g = torch.empty(1, dtype=torch.float32, device=dev)
        self.sf = torch.empty(L.fp4_mma_scales_bytes(M, K // 16), dtype=u8, device=dev)
        self.d = torch.empty((M, N), dtype=torch.float32, device=dev)
        st = torch.cuda.current_stream().cuda_stream
        P = lambda t: t.data_ptr()  # noqa: E731
        self.calls = [
            (L.fp4_tensor_amax, (P(x), fp4.BF16, self.n, P(self.amax), P(self.ws), self.ws.numel(), P(self.status), st)),
            (L.fp4_nvfp4_quantize_with_amax, (P(x), fp4.BF16, M, K, P(self.amax), P(self.p), P(self.s), P(self.g),
                                              P(self.status), st)),
            (L.fp4_scales_to_mma_layout, (P(self.s), M, K // 16, P(self.sf), st)),
            (L.fp4_nvfp4_gemm, (P(self.p), P(self.sf), P(self.g), P(qw.packed), P(self.w_sf), P(qw.global_scale),
                                M, N, K, P(self.d), P(self.status), st)),
        ]
        self.results = [self.d, self.status]

    step = Path.step
    check_status = Path.check_status

    def twin(self, x2: torch.Tensor) -> "GemmPath":
        return GemmPath(x2, shared=self)


def e2e_serial(path, x, x_host, steps: int, flush_l2) -> tuple[float, str]:
    """Milliseconds for `steps` steps, each on its own: L2 flush, upload of x
    from pinned memory, the step, download of every result, wait."""
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in path.results]
    ms = 0.0
    for k in range(steps + 2):
        flush_l2()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        x.copy_(x_host, non_blocking=True)
        path.step()
        for h, t in zip(host_out, path.results):
            h.copy_(t, non_blocking=True)
        e1.record()
        e1.synchronize()
        if int(host_out[-1].item()) != 0:
            raise RuntimeError("device status set during the end-to-end run")
        if k >= 2:
            ms += e0.elapsed_time(e1)
    return ms, "serial: upload, step, download, wait; L2 flushed before each step"


def e2e_pipelined(path, x, x_host, steps: int) -> tuple[float, str]:
    """Milliseconds for `steps` steps streamed the way a caller feeds batches:
    two device input buffers and two sets of outputs; step k's upload runs on
    an upload stream, its kernels on the compute stream, its downloads on a
    download stream, so the upload of step k+1 overlaps the kernels and the
    download of step k (the link is full duplex).  Every step uploads its
    whole input from pinned host memory and downloads every result; one
    event pair on the device spans the first upload to the last download."""
    paths = [path, path.twin(torch.empty_like(x))]
    xs = [x, paths[1].x]
    outs = [[torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in p.results] for p in paths]
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()

    def run(n: int) -> float:
        ev = [[torch.cuda.Event() for _ in range(n)] for _ in range(3)]  # upload, compute, download
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(up)
        for k in range(n):
            b = k % 2
            if k >= 2:
                up.wait_event(ev[1][k - 2])  # the kernels of step k-2 have read xs[b]
            with torch.cuda.stream(up):
                xs[b].copy_(x_host, non_blocking=True)
            ev[0][k].record(up)
            comp.wait_event(ev[0][k])
            if k >= 2:
                comp.wait_event(ev[2][k - 2])  # outputs of step k-2 downloaded
            paths[b].step()
            ev[1][k].record(comp)
            down.wait_event(ev[1][k])
            with torch.cuda.stream(down):
                for h, t in zip(outs[b], paths[b].results):
                    h.copy_(t, non_blocking=True)
            ev[2][k].record(down)
        end.record(down)
        end.synchronize()
        for o in outs:
            if int(o[-1].item()) != 0:
                raise RuntimeError("device status set during the end-to-end run")
        return start.elapsed_time(end)

    run(4)  # warm-up: streams, pinned buffers, the twin's first launches
    return run(steps), ("double-buffered: upload of step k+1 (upload stream) overlaps the kernels (compute "
                        "stream) and the download (download stream) of step k; every step's input uploaded "
                        "from pinned host memory, every result downloaded; no L2 flush between steps")


def e2e_layered(path, x, x_host, steps: int) -> tuple[float, str]:
    """Milliseconds for `steps` steps over the weight set, each streamed layer
    by layer the way a caller quantising a model feeds it: layer l's
    matrices are uploaded on an upload stream, their five grouped calls run
    on the compute stream once the upload is in, and their packed codes and
    scale bytes go back on a download stream, so that uploads, kernels and
    downloads of different layers overlap (the link is full duplex).  Every
    step uploads the whole set from pinned host memory and downloads every
    result (the per-matrix g and the status word after the last layer); one
    event pair on the device spans each step, and the steps are timed one
    after another."""
    host_out = [torch.empty(t.shape, dtype=t.dtype, pin_memory=True) for t in path.results]
    host_of = {id(t): h for t, h in zip(path.results, host_out)}
    comp = torch.cuda.current_stream()
    up, down = torch.cuda.Stream(), torch.cuda.Stream()
    n_layers = len(path.layers)

    def one() -> float:
        ev_up = [torch.cuda.Event() for _ in range(n_layers)]
        ev_c = [torch.cuda.Event() for _ in range(n_layers)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        start.record(up)
        comp.wait_event(start)
        down.wait_event(start)
        for l, (e0, e1, calls) in enumerate(path.layers):
            with torch.cuda.stream(up):
                x[e0:e1].copy_(x_host[e0:e1], non_blocking=True)
            ev_up[l].record(up)
            comp.wait_event(ev_up[l])
            for fn, args in calls:
                st = fn(*args)
                if st != 0:
                    raise path.fp4.FP4Error(st, fn.__name__)
            ev_c[l].record(comp)
            down.wait_event(ev_c[l])
            with torch.cuda.stream(down):
                for t, sl in path.layer_outputs(e0, e1):
                    host_of[id(t)][sl].copy_(t[sl], non_blocking=True)
        with torch.cuda.stream(down):
            for t in (path.nv_g, path.status):
                host_of[id(t)].copy_(t, non_blocking=True)
        end.record(down)
        end.synchronize()
        if int(host_of[id(path.status)].item()) != 0:
            raise RuntimeError("device status set during the end-to-end run")
        return start.elapsed_time(end)

    one()  # warm-up: streams, pinned buffers
    ms = sum(one() for _ in range(steps))
    return ms, ("layer-streamed: each step uploads the set layer by layer (upload stream), runs the five grouped "
                "calls on each layer's seven matrices once its upload is in (compute stream) and downloads the "
                "layer's codes and scale bytes (download stream), so that the three overlap across layers; every "
                "element uploaded from pinned host memory and every result downloaded each step")


def max_over_ranks(values: list[float], device, world: int) -> list[float]:
    """Element-wise max of per-rank timings (one all-reduce; identity at N=1)."""
    if world == 1:
        return list(values)
    t = torch.tensor(values, dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return t.tolist()


class L2Flush:
    """Between timed steps: write a buffer larger than L2 (evicting x and the
    outputs), then read a second one, so that the dirty lines of the write
    are written back before the next step and L2 starts clean and cold."""

    def __init__(self, mib: int, device):
        self.w = torch.empty(mib << 20, dtype=torch.uint8, device=device) if mib else None
        self.r = torch.ones((mib // 2) << 18, dtype=torch.int32, device=device) if mib else None

    def __call__(self):
        if self.w is not None:
            self.w.zero_()
            self.r.sum()


# Steps of each pass when not given: about a second of timed work.
DEFAULT_STEPS = {MODEL_WEIGHTS: 40}
DEFAULT_E2E_STEPS = {MODEL_WEIGHTS: 4}


def step_counts(args) -> tuple[int, int, int]:
    """(timed steps, per-kernel breakdown steps, end-to-end steps)."""
    K = args.steps if args.steps is not None else DEFAULT_STEPS.get(args.workload, 4000)
    Kb = max(3, min(K, args.breakdown_steps if args.breakdown_steps is not None else 500))
    Ke = max(3, min(K, args.e2e_steps if args.e2e_steps is not None else DEFAULT_E2E_STEPS.get(args.workload, 200)))
    return K, Kb, Ke


def run_ours(args, rank: int, world: int, local: int):
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    rows_mode = args.shard == "rows" and world > 1
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)
    if args.shard == "rows" and (args.workload == MODEL_WEIGHTS or args.workload == GEMM_WORKLOAD
                                 or args.workload in LAYOUT_WORKLOADS):
        raise SystemExit("--shard rows takes a single-tensor workload (the weight set shards by matrix: "
                         "use --shard replicas)")
    w = WORKLOADS[args.workload] if rows_mode else workloads.for_rank(WORKLOADS[args.workload], rank)
    if args.workload == MODEL_WEIGHTS:
        path = GroupedPath(dev, rank, args.model_layers)
        if args.model_layers != workloads.MODEL_LAYERS:  # a profiling-sized subset of the set
            w = dataclasses.replace(w, rows=path.n // w.cols,
                                    name=f"{w.name}@{args.model_layers}-layers")
        x = path.x
        x_host = torch.empty(x.shape, dtype=x.dtype, pin_memory=True)
        x_host.copy_(x)
    else:
        full = workloads.generate(w)
        if rows_mode:  # this rank's rows of the one tensor
            r0, r1 = shard_rows(w.rows, world, rank)
            full = full[r0:r1]
        x_host = full.contiguous().pin_memory()
        del full
        x = x_host.to(dev, non_blocking=False)
        kind = LAYOUT_WORKLOADS.get(args.workload)
        if args.workload == GEMM_WORKLOAD:
            path = GemmPath(x, workloads.generate(workloads.for_rank(workloads.GEMM_W, rank), device=dev))
        elif kind:
            path = LayoutPath(x, kind)
        else:
            path = ShardedPath(x) if rows_mode else Path(x)
    flush_l2 = L2Flush(args.flush_mib, dev)
    nops = len(path.OPS)
    K, Kb, Ke = step_counts(args)

    warmup = max(args.warmup, 3)
    for _ in range(warmup):
        flush_l2()
        path.step()
    torch.cuda.synchronize()
    path.check_status()

    # ---- timed region: K steps, one event pair around each step -----------
    # Nothing is recorded between the launches of a step: an event between
    # two kernels makes each launch wait for its predecessor's completion,
    # where the programmatic serialisation lets it launch as the
    # predecessor's CTAs retire.
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    clocks = ClockSampler(local)
    clocks.start()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    clocks.mark(True)
    wall0 = time.perf_counter()
    for k in range(K):
        flush_l2()
        evs[k][0].record()
        path.step()
        evs[k][1].record()
    torch.cuda.synchronize()
    wall = time.perf_counter() - wall0
    clocks.mark(False)
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    path.check_status()
    total_ms = sum(e0.elapsed_time(e1) for e0, e1 in evs)

    # ---- per entry point: a second pass with an event after every launch ---
    bevs = [[torch.cuda.Event(enable_timing=True) for _ in range(nops + 1)] for _ in range(Kb)]
    for k in range(Kb):
        flush_l2()
        bevs[k][0].record()
        path.step(bevs[k])
    torch.cuda.synchronize()
    path.check_status()
    per_op_ms = [sum(bevs[k][i].elapsed_time(bevs[k][i + 1]) for k in range(Kb)) for i in range(nops)]

    # ---- end to end through the same calls from pinned host memory ---------
    h2d = x.numel() * x.element_size()
    d2h = sum(t.numel() * t.element_size() for t in path.results)
    if hasattr(path, "layers"):
        e2e_ms, e2e_schedule = e2e_layered(path, x, x_host, Ke)
    elif hasattr(path, "twin"):
        e2e_ms, e2e_schedule = e2e_pipelined(path, x, x_host, Ke)
    else:
        e2e_ms, e2e_schedule = e2e_serial(path, x, x_host, Ke, flush_l2)

    total_ms, e2e_ms, *per_op_ms = max_over_ranks([total_ms, e2e_ms] + per_op_ms, dev, world)
    if world > 1:
        torch.distributed.destroy_process_group()
    if rank != 0:
        return

    # whole-job elements: every rank's own tensor (replicas), or the one
    # tensor the ranks share (rows)
    n_all = w.numel if rows_mode else w.numel * world
    w_rank = dataclasses.replace(w, rows=x.shape[0]) if rows_mode else w  # rank 0's share, per kernel
    value = n_all * K / (total_ms / 1e3)
    pk = peaks()
    ab = algorithmic_bytes(w_rank)
    if args.workload == GEMM_WORKLOAD:  # operands, their scales and the fp32 output
        M_, N_, K_ = path.M, path.N, path.K
        ab["nvfp4_gemm"] = (M_ + N_) * (K_ // 2 + K_ // 16) + 4 * M_ * N_
    kernels = {}
    for name, ms in zip(path.OPS, per_op_ms):
        us = ms / Kb * 1e3
        entry = {"us": round(us, 3), "share": round(ms / sum(per_op_ms), 4)}
        if name in ab:
            gbs = ab[name] / (us * 1e-6) / 1e9
            entry.update(gbs=round(gbs, 1), frac_hbm=round(gbs / pk["hbm_gbs"], 4))
        kernels[name] = entry
    dom = max((k for k in kernels if k in ab), key=lambda k: kernels[k]["us"])
    n_cand = search_candidate_count(x, path.ss_g.item()) if dom == "scale_search" else None
    step_desc = ("amax, nvfp4 quantize, mxfp4 quantize, nvfp4 dequantize (bf16), mxfp4 dequantize (bf16), "
                 "nvfp4 64-candidate scale search")
    if rows_mode:
        step_desc = "per-rank amax, max all-reduce of the 4-byte amax (NCCL), then " + step_desc[len("amax, "):]
    if args.workload in LAYOUT_WORKLOADS:
        step_desc = {"columns": "amax, column-wise nvfp4 quantize (Q(W^T)), column-wise mxfp4 quantize, "
                                "nvfp4 and mxfp4 dequantize of the transposed padded layouts (bf16)",
                     "padded": "amax, nvfp4 and mxfp4 quantize of rows padded to whole blocks, nvfp4 and "
                               "mxfp4 dequantize back to the logical shape (bf16)",
                     "variants": "amax, nvfp4 four-over-six quantize (its own amax + the two-candidate kernel), "
                                 "mxfp4 quantize with the ceil scale rule, nvfp4 and mxfp4 dequantize (bf16)"
                     }[LAYOUT_WORKLOADS[args.workload]]
    if args.workload == GEMM_WORKLOAD:
        step_desc = ("activation amax, nvfp4 quantize, scales to the MMA layout, tcgen05 block-scaled NVFP4 GEMM "
                     "D [8192, 4096] fp32 with the weight [4096, 14336] quantised once before timing")
    if args.workload == MODEL_WEIGHTS:
        step_desc = ("grouped over all 224 matrices (one kernel per pass): per-matrix amax, nvfp4 quantize "
                     "(per-matrix g), mxfp4 quantize, nvfp4 dequantize (bf16), mxfp4 dequantize (bf16)")
    gemm_mnk = (path.M, path.N, path.K) if args.workload == GEMM_WORKLOAD else None
    if gemm_mnk:
        dom = "nvfp4_gemm"  # the tensor-core kernel is the one this workload is about
    if LAYOUT_WORKLOADS.get(args.workload) == "variants" and dom == "nvfp4_quantize":
        # four over six: two screened candidates per block, ALU-bound like the search
        n_cand = 2 * (w_rank.numel // 16)
        roof = roofline_for("scale_search", kernels[dom], w_rank, pk, n_cand)
        roof["kernel"] = "nvfp4_quantize_four_over_six"
        roof["work"] = roof["work"].replace("distinct candidates", "candidates (2 per block)")
    else:
        roof = roofline_for(dom, kernels[dom], w_rank, pk, n_cand, gemm_mnk)
    line = {
        "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": K,
        "warmup": warmup, "ms_per_step": total_ms / K, "higher_is_better": True,
        "scaling": "strong" if rows_mode else "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name if world == 1 or rows_mode else WORKLOADS[args.workload].name,
                   "description": WORKLOADS[args.workload].description,
                   "shape": ([[r, c] for r, c in workloads.MODEL_MATRICES] if args.workload == MODEL_WEIGHTS
                             else [w.rows, w.cols]),
                   "input_dtype": str(w.dtype).replace("torch.", ""),
                   "arithmetic": "fp32 (element quotients, block-scale decisions and dequantised products)",
                   "step": step_desc,
                   "l2": (f"flushed between steps outside the timed events ({args.flush_mib} MiB write, "
                          f"then {args.flush_mib // 2} MiB read)" if args.flush_mib else "not flushed") +
                         (f"; input {w.numel * w.dtype.itemsize / 1e9:.1f} GB, larger than the 126 MB L2"
                          if w.numel * w.dtype.itemsize > 126e6 else ""),
                   "parallelism": (f"rows split over {world} ranks, one max all-reduce of the amax per step"
                                   if rows_mode else
                                   f"replicas x{world} (independent tensors)" if world > 1 else "single GPU")},
        "hbm_gbs_step": sum(ab[o] for o in path.OPS if o in ab) * (world if rows_mode else 1)
                        / (total_ms / K * 1e-3) / 1e9,
        "kernels": kernels,
        "kernels_timing": (f"second pass of {Kb} steps, L2 flushed between steps, an event after every launch: "
                           "the events serialise the launches, so each time includes its own launch and ramp "
                           "and the times add up to more than ms_per_step"),
        "roofline": roof,
        "e2e": {"value": n_all * Ke / (e2e_ms / 1e3), "unit": "elements/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "schedule": e2e_schedule},
        "gpu_launches": path.LAUNCHES * K,
        "clocks": clk,
        "wall_s_timed": wall,
    }
    if dom != "nvfp4_quantize" and "nvfp4_quantize" in kernels and "nvfp4_quantize" in ab and not gemm_mnk \
            and LAYOUT_WORKLOADS.get(args.workload) != "variants":
        line["roofline_nvfp4_quantize"] = roofline_for("nvfp4_quantize", kernels["nvfp4_quantize"], w_rank, pk)
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, budget_s=args.cpu_budget)
    print(json.dumps(line), flush=True)


def search_candidate_count(x: torch.Tensor, g: float) -> int:
    """Number of distinct scale candidates the search definition leaves after
    merging duplicates, summed over the blocks of x: the candidates of a block
    are the contiguous E4M3 codes from round(0.70 A_b/(6g)) to round(A_b/(6g)).
    Counted with torch (fp32 quotients, torch's E4M3 rounding) once per
    workload, outside the timed region; it sizes the work, not the output."""
    ab = x.float().reshape(-1, 16).abs().amax(dim=1).double()
    t_hi = (ab / (6.0 * g)).clamp(max=448.0).float()
    t_lo = (ab * 147.0 / (1260.0 * g)).clamp(max=448.0).float()
    c_hi = t_hi.to(torch.float8_e4m3fn).view(torch.uint8).long()
    c_lo = t_lo.to(torch.float8_e4m3fn).view(torch.uint8).long()
    return int((c_hi - c_lo + 1).sum().item())


# fp32 operations of one candidate-element evaluation of the search: quotient
# (one multiply by a reciprocal), round to the E2M1 grid, decode, two
# reconstruction multiplies, subtract, square-accumulate.
SEARCH_OPS_PER_EVAL = 7


def traffic_sources(workload: str) -> tuple:
    """Sources beyond KERNEL_SOURCES whose kernels a workload's traffic
    figures were captured from (the layout and GEMM kernels)."""
    if workload in LAYOUT_WORKLOADS:
        return tuple(LAYOUT_SOURCES)
    if workload == GEMM_WORKLOAD:
        return tuple(GEMM_SOURCES)
    return ()


def roofline_for(name: str, k: dict, w: workloads.Workload, pk: dict, n_cand: int | None = None,
                 gemm_mnk=None) -> dict:
    # DRAM bytes per launch from an ncu capture (profiles/traffic.json), used
    # only while the kernel sources are the ones it was captured from
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            t = json.load(f)
        ent = t.get("workloads", {}).get(w.name, {}).get(name)
        if ent and ent.get("source_hash") == kernel_source_hash(traffic_sources(w.name)):
            traffic = ent.get("bytes_per_launch")
    if name == "nvfp4_gemm" and gemm_mnk:
        # tensor-bound: 2 M N K flops per launch against the FP4 dense peak,
        # taken as the measured bf16 GEMM peak times the nominal FP4 / bf16
        # ratio (9 / 2.25 PFLOP/s dense)
        M, N, K = gemm_mnk
        peak = pk["bf16_tflops"] * 4.0
        achieved = 2.0 * M * N * K / (k["us"] * 1e-6) / 1e12
        return {"bound": "tensor", "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": "TFLOP/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": name,
                "work": f"2 x {M} x {N} x {K} flops",
                "peak_source": f"measured bf16 {pk['bf16_tflops']:.1f} TFLOP/s x 4 (nominal FP4 / bf16 ratio)"}
    if name == "scale_search" and n_cand:
        # ALU-bound: fp32 lane operations of the distinct candidate
        # evaluations per second, against SMs x 128 FP32 lanes x max SM clock.
        sms = torch.cuda.get_device_properties(torch.cuda.current_device()).multi_processor_count
        peak = sms * 128 * pk["sm_max_mhz"] * 1e6 / 1e12
        achieved = n_cand * 16 * SEARCH_OPS_PER_EVAL / (k["us"] * 1e-6) / 1e12
        return {"bound": "alu", "achieved": round(achieved, 3), "peak": round(peak, 2), "unit": "Tops/s",
                "frac": round(achieved / peak, 4), "traffic": traffic, "kernel": name,
                "work": f"{n_cand} distinct candidates x 16 elements x {SEARCH_OPS_PER_EVAL} fp32 ops",
                "peak_source": f"{sms} SMs x 128 FP32 lanes x {pk['sm_max_mhz']:.0f} MHz ({pk['source']})"}
    return {"bound": "hbm", "achieved": k["gbs"], "peak": pk["hbm_gbs"], "unit": "GB/s",
            "frac": k["frac_hbm"], "traffic": traffic, "kernel": name, "peak_source": pk["source"]}


# ------------------------------------------------------- CPU oracle legs --

def _oracle_step(xs, search: bool = True):
    import oracle
    p, s, g = oracle.nvfp4_quantize(xs)
    pm, sm = oracle.mxfp4_quantize(xs)
    R, C = xs.shape
    oracle.nvfp4_dequantize(p, s, g, R, C)
    oracle.mxfp4_dequantize(pm, sm, R, C)
    if search:
        oracle.nvfp4_scale_search(xs)


def _oracle_layout_step(xs, kind: str):
    """The layout and variant workloads' step on the oracle: four over six
    and the MXFP4 ceil rule, or column-wise or row-padded quantisation in
    both formats, then the dequantisations."""
    import oracle
    R, C = xs.shape
    if kind == "variants":
        p, s, g, _ = oracle.nvfp4_quantize_four_over_six(xs)
        pm, sm = oracle.mxfp4_quantize_rule(xs, oracle.MX_CEIL)
        oracle.nvfp4_dequantize(p, s, g, R, C)
        oracle.mxfp4_dequantize(pm, sm, R, C)
        return
    if kind == "columns":
        p, s, g = oracle.nvfp4_quantize_columns(xs)
        pm, sm = oracle.mxfp4_quantize_columns(xs)
        R, C = C, R
    else:
        p, s, g = oracle.nvfp4_quantize_padded(xs)
        pm, sm = oracle.mxfp4_quantize_padded(xs)
    oracle.nvfp4_dequantize_padded(p, s, g, R, C)
    oracle.mxfp4_dequantize_padded(pm, sm, R, C)


_GEMM_W_SLICE = 256  # weight rows the oracle multiplies by (of 4096)


def _oracle_gemm_step_factory():
    """The GEMM workload on the oracle: quantise the sample rows of the
    activation and multiply them by the first 256 rows of the quantised
    weight (the weight is quantised once, before timing, as in the GPU
    arm)."""
    import oracle
    wsl = workloads.as_oracle_array(workloads.generate(workloads.GEMM_W))[:_GEMM_W_SLICE]
    wp, wsc, wg = oracle.nvfp4_quantize(np.ascontiguousarray(wsl))

    def step(xs):
        p, s, g = oracle.nvfp4_quantize(xs)
        oracle.nvfp4_gemm(p, s, g, wp, wsc, wg, xs.shape[0], _GEMM_W_SLICE, xs.shape[1])
    return step


def oracle_sample_source(w: workloads.Workload):
    """(tensor the CPU legs sample rows from, the step on a row sample, what
    the sample is): the workload itself, or for the whole weight set its
    first matrix (same distribution; the set is too large to draw on the
    host)."""
    if w.name.startswith(MODEL_WEIGHTS):
        return (workloads.generate(workloads.model_matrix(0, 0)), lambda xs: _oracle_step(xs, False),
                "its first matrix")
    kind = LAYOUT_WORKLOADS.get(w.name)
    if kind:
        return workloads.generate(w), lambda xs: _oracle_layout_step(xs, kind), w.name
    if w.name == GEMM_WORKLOAD:
        return (workloads.generate(w), _oracle_gemm_step_factory(),
                f"{w.name}, times the first {_GEMM_W_SLICE} of the 4096 weight rows")
    return workloads.generate(w), _oracle_step, w.name


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


def time_oracle_rows(step, xo, r0: int, rows: int, threads: int) -> float:
    """Seconds for `step` over rows [r0, r0 + rows) of xo, split into
    `threads` contiguous row ranges run concurrently, one per thread (the
    oracle is C called through ctypes, which releases the GIL for the
    duration of each call).  The oracle itself is unchanged: each thread
    runs the plain single-threaded code on its own rows."""
    import concurrent.futures
    bounds = [r0 + shard_rows(rows, threads, t)[0] for t in range(threads)] + [r0 + rows]
    parts = [np.ascontiguousarray(xo[bounds[t]:bounds[t + 1]]) for t in range(threads)]
    parts = [p for p in parts if p.shape[0]]
    t0 = time.perf_counter()
    if len(parts) == 1:
        step(parts[0])
    else:
        with concurrent.futures.ThreadPoolExecutor(max_workers=len(parts)) as ex:
            for f in [ex.submit(step, p) for p in parts]:
                f.result()
    return time.perf_counter() - t0


def _rows_for(step, xo, budget_s: float, threads: int) -> int:
    """Rows that keep one timing of `step` on `threads` threads near
    budget_s, from a 32-row probe on one thread."""
    R = xo.shape[0]
    t_row = time_oracle_rows(step, xo, 0, min(R, 32), 1) / min(R, 32)
    return int(max(min(threads, R), min(R, budget_s * threads / max(t_row, 1e-6))))


def cpu_baseline(w: workloads.Workload, budget_s: float = 8.0) -> dict:
    """The oracle as it stands (plain single-threaded C) on bounded row
    samples of the same workload, the same steps, in elements/s: first on
    one core, then on every host core at once (one row range per thread)."""
    import oracle
    oracle.build()
    x, step, what = oracle_sample_source(w)
    xo = workloads.as_oracle_array(x)
    R, C = xo.shape
    rows1 = _rows_for(step, xo, budget_s, 1)
    dt1 = time_oracle_rows(step, xo, 0, rows1, 1)
    cores = host_cores()
    rowsn = min(R, rows1 * cores)
    reps, dtn = 0, 0.0
    while reps == 0 or dtn < budget_s / 2:  # repeat a sample the tensor's rows cap
        dtn += time_oracle_rows(step, xo, 0, rowsn, cores)
        reps += 1
    return {"value": reps * rowsn * C / dtn, "unit": "elements/s", "cores": cores, "kind": "oracle",
            "sample": (f"first {rowsn} of {R} rows ({rowsn * C} elements) of {what}, whole step, split over "
                       f"{cores} threads, {reps} time(s), {dtn:.1f} s"),
            "one_core": {"value": rows1 * C / dt1, "cores": 1,
                         "sample": f"first {rows1} rows ({rows1 * C} elements), {dt1:.1f} s"},
            "cpu": _cpu_model()}


def _cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank: int, world: int):
    """--impl reference: the CPU oracle on every host core, rank 0 only;
    each step a bounded row sample of the workload split into one row
    range per core (the plain single-threaded oracle on each)."""
    if rank != 0:
        return
    import oracle
    oracle.build()
    w = WORKLOADS[args.workload]
    x, step, what = oracle_sample_source(w)
    xo = workloads.as_oracle_array(x)
    R, C = xo.shape
    cores = host_cores()
    total_budget = 120.0
    steps = args.steps if args.steps is not None else 20
    warm = max(args.warmup, 0)
    rows = min(R, _rows_for(step, xo, total_budget / (steps + warm), cores))
    for _ in range(warm):
        time_oracle_rows(step, xo, 0, rows, cores)
    dt = 0.0
    for k in range(steps):
        r0 = (k * rows) % max(1, R - rows + 1)
        dt += time_oracle_rows(step, xo, r0, rows, cores)
    value = rows * C * steps / dt
    line = {
        "metric": METRIC, "value": value, "unit": "elements/s", "n_gpus": world, "steps": steps,
        "warmup": warm, "ms_per_step": dt / steps * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic", "impl": "reference",
        "config": {"workload": w.name, "description": w.description, "shape": [w.rows, w.cols]},
        "cpu_baseline": {"value": value, "unit": "elements/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows} rows x {C} per step, split over {cores} threads "
                                   f"(bounded sample of {what})",
                         "cpu": _cpu_model()},
        "e2e": {"value": value, "unit": "elements/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


import numpy as np  # noqa: E402  (used by the reference leg)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 40 on the weight set, 4000 on the single tensors)")
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default=DEFAULT_WORKLOAD)
    ap.add_argument("--e2e-steps", type=int, default=None,
                    help="steps of the end-to-end pass (default: 4 on the weight set, 200 otherwise)")
    ap.add_argument("--breakdown-steps", type=int, default=None,
                    help="steps of the per-entry-point pass (events between launches)")
    ap.add_argument("--cpu-budget", type=float, default=8.0,
                    help="seconds of each CPU-baseline leg (one core, then all cores)")
    ap.add_argument("--shard", choices=["replicas", "rows"], default="replicas",
                    help="multi-GPU mode: each rank its own tensor, or one tensor split by rows")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--model-layers", type=int, default=workloads.MODEL_LAYERS,
                    help="layers of the 7B weight set in model-7b-weights-bf16 (fewer only for profiler runs)")
    ap.add_argument("--flush-mib", type=int, default=512,
                    help="L2 flush size between steps (0 = no flush, for profiler runs only)")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local)


if __name__ == "__main__":
    main()
