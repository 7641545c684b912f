#!/usr/bin/env python
"""Benchmark of the blockwise FP8 weight quantizer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload qwen3_8b_model|qwen3_8b_layer|qwen3_8b_layer_f32|moe_layer|
                                small|act_1x128|blk_64x64|qkv|ragged|edge] [--repeat R]
                    [--path auto|vector|tma|generic] [--mode grouped|per_layer|per_tensor]
                    [--op quantize|dequantize|tensor_scale|shard] [--pdl on|off]

A step is one pass of the whole quantizer over the workload: by default the
full Qwen3-8B-shaped weight set (36 layers x q,k,v,o,gate,up,down = 252 bf16
tensors, 6.95e9 elements, 13.9 GB in + 6.95 GB out) quantized to e4m3fn with
128x128 blocks in ONE grouped call of the C ABI (fp8bq_quantize_batched).

Metric: GB/s of algorithmic bytes (input read + e4m3 write + fp32 descales),
whole job over all ranks, timed with CUDA events on the launching stream
around K steps issued back to back (a step's kernels may start while the
previous step's drain: programmatic dependent launch, --pdl), the
inputs already resident in HBM; the inputs (13.9 GB) are far larger than L2
(126 MB), so no flush is needed between steps.  `e2e` is the same metric
with the inputs in pinned host memory and the outputs copied back to host
memory inside the timed region, one C-ABI call per layer, the copies of
neighbouring layers overlapping the compute.

N > 1 (torchrun, one process per GPU): every rank quantizes its own replica of
the weight set (weak scaling; no collective on the data path; the host inputs
are generated once per node into shared memory).  Timing is the max over
ranks.

--impl reference times the CPU oracle (single thread) on a bounded sample of
the same workload: one tensor per step, cycling through the weight set.
"""
from __future__ import annotations

import argparse
import ctypes
import datetime
import hashlib
import json
import os
import platform
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "blockwise FP8 quant GB/s (bytes in+out) and % of B200 HBM peak, 1 GPU"
FALLBACK_HBM_GBS = 6650.0
# the sources of the TMA kernels, whose DRAM traffic profiles/traffic.txt records
KERNEL_SOURCES = ["blockwise_fp8_weight_b200/csrc/fp8bq_tma.cu",
                  "blockwise_fp8_weight_b200/csrc/fp8bq_tile.cuh",
                  "blockwise_fp8_weight_b200/csrc/fp8bq_device.cuh",
                  "blockwise_fp8_weight_b200/csrc/fp8bq_internal.h"]
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.txt")
PATHS = {"auto": 0, "vector": 1, "tma": 2, "generic": 3}


# ------------------------------------------------------------------ distributed plumbing


def dist_env() -> tuple[int, int, int]:
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("LOCAL_RANK", "0")),
            int(os.environ.get("WORLD_SIZE", "1")))


class Dist:
    """Process-group plumbing: barrier and max-over-ranks of a scalar."""

    def __init__(self, world: int, backend: str, device=None):
        self.world = world
        self.device = device
        if world > 1:
            import torch.distributed as dist
            dist.init_process_group(backend, timeout=datetime.timedelta(seconds=600))
            self.dist = dist

    def barrier(self):
        if self.world > 1:
            if self.device is not None:
                self.dist.barrier(device_ids=[self.device.index])
            else:
                self.dist.barrier()

    def max(self, v: float) -> float:
        if self.world == 1:
            return v
        import torch
        t = torch.tensor([v], dtype=torch.float64, device=self.device or "cpu")
        self.dist.all_reduce(t, op=self.dist.ReduceOp.MAX)
        return float(t.item())

    def close(self):
        if self.world > 1:
            self.dist.destroy_process_group()


def aggregate(bytes_per_step: int, steps: int, world: int, max_elapsed_s: float) -> float:
    """Whole-job GB/s: bytes every rank moved over all timed steps / slowest rank's time."""
    return bytes_per_step * steps * world / max_elapsed_s / 1e9


# ------------------------------------------------------------------ workload


def workload(name: str):
    from synth import TensorSpec
    from synth import workloads as W
    if name == "qwen3_8b_model":
        return W.qwen3_8b_model(), ("Qwen3-8B-shaped full weight set: 36 layers x (q,k,v,o,"
                                    "gate,up,down) bf16, block 128x128, one grouped launch")
    if name == "qwen3_8b_layer":
        return W.qwen3_8b_layer(0, seed=1), ("one Qwen3-8B-shaped layer: 7 bf16 linear weights, "
                                             "block 128x128, one grouped launch")
    if name == "qwen3_8b_layer_f32":
        specs = W.qwen3_8b_layer(0, seed=1)
        for sp in specs:
            sp.dtype = "f32"
        return specs, ("one Qwen3-8B-shaped layer in fp32 (7 linear weights), block 128x128, "
                       "one grouped launch")
    if name == "moe_layer":
        return W.moe_layer(0), ("one Qwen3-30B-A3B-style MoE layer: q,k,v,o + 128-expert w13 "
                                "and w2 stacks, bf16, block 128x128, one grouped launch")
    if name == "small":
        return W.small(), "256x384 bf16, 2x3 blocks of 128x128"
    if name == "qkv":
        return W.qkv_activations(), ("Q/K/V activations of one Qwen3-8B-shaped attention layer, "
                                     "16384 tokens, bf16 (per-tensor scale recalibration)")
    if name == "ragged":
        sp = [t for t in W.edge() if t.name == "edge.bf16.4000x4100"]
        return sp, "bf16 4000x4100 (rows only 8-byte aligned), block 128x128, Student-t(3) x 0.02"
    if name == "edge":
        return W.edge(), ("ragged and small-block edge set in one grouped call: bf16 and fp32 "
                          "4000x4100, 130x129, 1x128, 12345x4096, 4000x4100 with ld 4164 "
                          "(block 128x128), bf16 16384x4096 with [1,128] and [64,64] blocks")
    if name.startswith("shape:"):  # shape:[BATCHx]MxN[:f32] -- one tensor, block 128x128
        dims, _, dt = name[6:].partition(":")
        v = [int(t) for t in dims.split("x")]
        batch, M, N = (v if len(v) == 3 else [1] + v)
        sp = TensorSpec(f"shape.{dims}", M, N, batch=batch, dtype=dt or "bf16", seed=5,
                        tensor_id=0, sigma=0.02)
        return [sp], f"one {sp.dtype} tensor [{batch}, {M}, {N}], block 128x128, N(0, 0.02)"
    if name in ("act_1x128", "blk_64x64"):
        sp = [t for t in W.edge() if t.name.endswith("b1x128" if name == "act_1x128" else "b64x64")]
        return sp, f"bf16 16384x4096, N(0,1) x row lognormal(0,1), blocks {sp[0].block}"
    raise SystemExit(f"unknown workload {name}")


def layers_of(specs) -> list[list[int]]:
    """Group tensor indices by layer (consecutive) for the per-layer e2e pipeline."""
    groups: list[list[int]] = []
    last = object()
    for i, sp in enumerate(specs):
        key = sp.meta.get("layer", 0)
        if key != last:
            groups.append([])
            last = key
        groups[-1].append(i)
    return groups


def align(v: int, a: int) -> int:
    return (v + a - 1) // a * a


class Layout:
    """Byte offsets of every tensor in the packed input / output buffers."""

    def __init__(self, specs):
        self.x_off, self.y_off, self.s_off = [], [], []
        xo = yo = so = 0
        for sp in specs:
            self.x_off.append(xo)
            self.y_off.append(yo)
            self.s_off.append(so)
            xo = align(xo + sp.numel_storage * sp.elem_bytes, 256)
            yo = align(yo + sp.numel, 256)
            so = align(so + sp.nblocks * 4, 256)
        self.x_bytes, self.y_bytes, self.s_bytes = xo, yo, so


def spec_digest(specs) -> str:
    h = hashlib.sha256()
    h.update(open(os.path.join(ROOT, "synth", "synth.c"), "rb").read())
    h.update(open(os.path.join(ROOT, "synth", "workloads.py"), "rb").read())
    for sp in specs:
        h.update(repr((sp.name, sp.M, sp.N, sp.batch, sp.row_stride, sp.dtype, sp.seed,
                       sp.tensor_id)).encode())
    return h.hexdigest()[:16]


def host_inputs(specs, lay: Layout, local_rank: int, dist: Dist, tag: str):
    """Generate the packed host inputs once per node into /dev/shm (shared by the
    ranks of a replica run); returns a writable numpy memmap."""
    from synth import workloads as W
    shm = "/dev/shm" if os.path.isdir("/dev/shm") else "/tmp"
    path = os.path.join(shm, f"fp8bq_bench_{tag}_{spec_digest(specs)}.bin")
    done = path + ".done"
    if local_rank == 0 and not os.path.exists(done):
        mm = np.memmap(path, dtype=np.uint8, mode="w+", shape=(lay.x_bytes,))
        base = mm.ctypes.data
        for sp, off in zip(specs, lay.x_off):
            W.materialize_into(sp, base + off)
        mm.flush()
        del mm
        open(done, "w").write("ok")
    dist.barrier()
    return np.memmap(path, dtype=np.uint8, mode="r+", shape=(lay.x_bytes,)), path


# ------------------------------------------------------------------ measurement helpers


class ClockSampler:
    """Samples SM clock, power and clock-event reasons with NVML while running."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
               0x8: "hw_slowdown", 0x20: "sync_boost", 0x40: "sw_thermal_slowdown",
               0x80: "hw_thermal_slowdown", 0x100: "hw_power_brake_slowdown",
               0x200: "display_clock_setting"}

    def __init__(self, torch_device, period_s=0.004):
        self.period = period_s
        self.samples, self.power, self.reason_samples = [], [], []
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        try:
            import pynvml
            pynvml.nvmlInit()
            import torch
            p = torch.cuda.get_device_properties(torch_device)
            bus = f"{p.pci_domain_id:08X}:{p.pci_bus_id:02X}:{p.pci_device_id:02X}.0"
            self.h = pynvml.nvmlDeviceGetHandleByPciBusId(bus)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _reasons_now(self):
        nv = self.nv
        f = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        return int(f(self.h))

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                self.reason_samples.append(self._reasons_now())
                self.power.append(self.nv.nvmlDeviceGetPowerUsage(self.h) / 1000.0)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.nv is not None:
            self._thr = threading.Thread(target=self._run, daemon=True)
            self._thr.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thr:
            self._thr.join()

    def summary(self) -> dict:
        if self.nv is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        n = len(self.reason_samples)
        frac = {name: round(sum(1 for r in self.reason_samples if r & bit) / n, 3)
                for bit, name in self.REASONS.items()
                if n and any(r & bit for r in self.reason_samples)}
        return {"sm_mhz": float(np.median(self.samples)) if self.samples else None,
                "sm_min_mhz": min(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "power_w_median": float(np.median(self.power)) if self.power else None,
                "reasons": sorted(frac), "reason_sample_fraction": frac}


def measured_peak() -> tuple[float, str]:
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(p))["hbm_gbs"])
        return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_digest() -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:16]


def traffic_for(workload_name: str, path: str, launches: int):
    """(DRAM bytes per launch, how they were obtained) from the committed ncu
    record of this workload (profiles/traffic.txt: "<workload> <path> <kernel
    sources sha256/16> <dram bytes per step> <source>", the source saying
    whether the step was captured or scaled from a smaller case), if it was
    taken on the current kernel sources; else (None, None)."""
    try:
        lines = open(TRAFFIC_FILE).read().splitlines()
    except OSError:
        return None, None
    for line in lines:
        f = line.split(maxsplit=4)
        if len(f) >= 4 and not line.startswith("#") and f[0] == workload_name and f[1] == path \
                and f[2] == kernel_digest():
            return float(f[3]) / max(launches, 1), (f[4] if len(f) > 4 else "captured")
    return None, None


# ------------------------------------------------------------------ arms


def run_reference(args) -> None:
    rank, _local, world = dist_env()
    if rank != 0:
        return
    import oracle
    from synth import workloads as W
    specs, desc = workload(args.workload)
    order = list(range(len(specs)))
    total_bytes = 0
    elapsed = 0.0
    for step in range(args.warmup + args.steps):
        sp = specs[order[step % len(order)]]
        x = W.materialize(sp)
        t0 = time.perf_counter()
        for b in range(sp.batch):
            xb = x[b * sp.batch_stride:(b + 1) * sp.batch_stride]
            oracle.quantize(xb, sp.M, sp.N, sp.row_stride, *sp.block)
        dt = time.perf_counter() - t0
        if step >= args.warmup:
            total_bytes += sp.algorithmic_bytes
            elapsed += dt
    value = total_bytes / elapsed / 1e9
    per_step = sum(sp.algorithmic_bytes for sp in specs)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_step / (value * 1e9) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": desc, "name": args.workload, "block": [128, 128]},
        "cpu_baseline": {"kind": "oracle", "value": value, "unit": "GB/s", "cores": 1,
                         "sample": f"one tensor of the workload per step, cycling from the "
                                   f"first; {args.steps} timed tensors after {args.warmup} warm-up; "
                                   f"single-threaded C oracle; {platform.processor() or 'cpu'}"},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "note": "ms_per_step extrapolates the sampled rate to the whole workload",
    }
    print(json.dumps(line), flush=True)


def build_descs(specs, lay: Layout, x_base: int, y_base: int, s_base: int, idx=None):
    import blockwise_fp8_weight_b200 as fq
    idx = range(len(specs)) if idx is None else idx
    arr = (fq.fp8bq_desc * len(idx))()
    for j, i in enumerate(idx):
        sp = specs[i]
        gm, gn = sp.grid
        d = arr[j]
        d.x = x_base + lay.x_off[i]
        d.y_u8 = y_base + lay.y_off[i]
        d.descale_f32 = s_base + lay.s_off[i]
        d.M, d.N, d.ld, d.batch = sp.M, sp.N, sp.row_stride, sp.batch
        d.x_batch_stride = sp.batch_stride
        d.y_batch_stride = sp.M * sp.N
        d.s_batch_stride = gm * gn
        d.dtype_in = fq.FP8BQ_BF16 if sp.dtype == "bf16" else fq.FP8BQ_F32
        d.block_m, d.block_n = sp.block
        d.reserved = 0
    return arr


def count_launches(arr) -> int:
    """Kernel launches of one fp8bq_quantize_batched call over `arr`, as the
    library plans them (fp8bq_launch_count)."""
    import blockwise_fp8_weight_b200 as fq
    n = fq.fp8bq_launch_count(arr, len(arr))
    if n < 0:
        raise RuntimeError("the library rejects this call")
    return n


def cpu_baseline(specs, host: np.ndarray, lay: Layout, seconds: float) -> dict:
    """The oracle as it stands, single-threaded, over whole tensors from the start
    of the workload until about `seconds` of CPU time has been spent."""
    import oracle
    done_bytes, done = 0, []
    t0 = time.perf_counter()
    for i, sp in enumerate(specs):
        x = host[lay.x_off[i]:lay.x_off[i] + sp.numel_storage * sp.elem_bytes].view(sp.np_dtype)
        for b in range(sp.batch):
            xb = np.ascontiguousarray(x[b * sp.batch_stride:(b + 1) * sp.batch_stride])
            oracle.quantize(xb, sp.M, sp.N, sp.row_stride, *sp.block)
        done_bytes += sp.algorithmic_bytes
        done.append(sp.name)
        if time.perf_counter() - t0 >= seconds:
            break
    dt = time.perf_counter() - t0
    cpu = platform.processor() or ""
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                cpu = line.split(":", 1)[1].strip()
                break
    except OSError:
        pass
    return {"value": done_bytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"first {len(done)} tensors of the workload ({done[0]} .. {done[-1]}), "
                      f"{done_bytes / 1e9:.2f} GB moved in {dt:.1f} s; host {cpu}, "
                      f"nproc {os.cpu_count()}"}


def run_ours(args) -> None:
    import torch
    import blockwise_fp8_weight_b200 as fq

    rank, local_rank, world = dist_env()
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    dist = Dist(world, "nccl", dev)
    specs, wl_desc = workload(args.workload)
    if args.only:  # a subset of the workload's tensors (by name)
        import re
        specs = [sp for sp in specs if re.search(args.only, sp.name)]
        if not specs:
            raise SystemExit(f"--only {args.only!r} matches no tensor of {args.workload}")
        wl_desc += f"; only the tensors matching {args.only!r}"
    if args.repeat > 1:  # the same tensor list args.repeat times, fresh values each time
        import dataclasses
        specs = [dataclasses.replace(sp, name=f"{sp.name}.r{k}", tensor_id=sp.tensor_id + 4096 * k,
                                     meta=dict(sp.meta, layer=k))
                 for k in range(args.repeat) for sp in specs]
        wl_desc += f", x{args.repeat} in one call"
    lay = Layout(specs)
    bytes_per_step = sum(sp.algorithmic_bytes for sp in specs)
    elements = sum(sp.numel for sp in specs)

    host, shm_path = host_inputs(specs, lay, local_rank, dist, args.workload)
    cudart = torch.cuda.cudart()
    hptr = host.ctypes.data
    reg = cudart.cudaHostRegister(hptr, lay.x_bytes, 0)
    pinned_in = int(reg) == 0
    host_t = torch.from_numpy(host)

    x_dev = torch.empty(lay.x_bytes, dtype=torch.uint8, device=dev)
    x_dev.copy_(host_t, non_blocking=False)
    y_dev = torch.empty(lay.y_bytes, dtype=torch.uint8, device=dev)
    s_dev = torch.empty(lay.s_bytes, dtype=torch.uint8, device=dev)
    table = build_descs(specs, lay, x_dev.data_ptr(), y_dev.data_ptr(), s_dev.data_ptr())
    n = len(table)
    assert fq.fp8bq_set_path(PATHS[args.path]) == fq.FP8BQ_OK
    assert fq.fp8bq_set_pdl(args.pdl == "on") == fq.FP8BQ_OK
    L = fq.lib()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    # grouped: the whole list in one call; per_layer: one call per layer;
    # per_tensor: one call per tensor (the pages' quant_weights loop)
    if args.mode == "grouped":
        calls = [table]
    elif args.mode == "per_layer":
        calls = [build_descs(specs, lay, x_dev.data_ptr(), y_dev.data_ptr(), s_dev.data_ptr(), g)
                 for g in layers_of(specs)]
    else:
        calls = [build_descs(specs, lay, x_dev.data_ptr(), y_dev.data_ptr(), s_dev.data_ptr(), [i])
                 for i in range(len(specs))]
    launches = sum(count_launches(c) for c in calls)

    def step():
        for c in calls:
            st = L.fp8bq_quantize_batched(c, len(c), sh)
            if st != 0:
                raise RuntimeError(fq.fp8bq_status_string(st))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    fq.check(fq.fp8bq_sync_status(stream), "warm-up")

    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(dev) as clk:
        torch.cuda.nvtx.range_push(f"fp8bq timed steps x{args.steps}")
        t_start.record(stream)
        for i in range(args.steps):   # back to back: no event between the steps' launches
            step()
        t_end.record(stream)
        torch.cuda.nvtx.range_pop()
        while not t_end.query():      # poll (not synchronize) so the sampler thread runs
            time.sleep(0.0005)
        torch.cuda.synchronize()
    dist.barrier()
    fq.check(fq.fp8bq_sync_status(stream), "timed steps")
    elapsed_s = t_start.elapsed_time(t_end) / 1e3
    max_elapsed = dist.max(elapsed_s)
    value = aggregate(bytes_per_step, args.steps, world, max_elapsed)

    if args.op in ("dequantize", "tensor_scale", "shard"):
        if args.op == "dequantize":
            run_dequant_op(args, specs, lay, y_dev, s_dev, dev, dist, world, rank, wl_desc)
        elif args.op == "shard":
            run_shard_op(args, specs, lay, x_dev, dev, dist, world, rank, wl_desc)
        else:
            run_scale_op(args, specs, lay, x_dev, dev, dist, world, rank, wl_desc)
        fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
        if pinned_in:
            cudart.cudaHostUnregister(hptr)
        del host_t, host
        dist.barrier()
        if local_rank == 0 and not args.keep_inputs:
            for pth in (shm_path, shm_path + ".done"):
                try:
                    os.remove(pth)
                except OSError:
                    pass
        dist.close()
        return

    # ---- end to end: inputs from pinned host memory, outputs back to host memory
    y_host = torch.empty(lay.y_bytes, dtype=torch.uint8, pin_memory=True)
    s_host = torch.empty(lay.s_bytes, dtype=torch.uint8, pin_memory=True)
    groups = layers_of(specs)
    tables = [build_descs(specs, lay, x_dev.data_ptr(), y_dev.data_ptr(), s_dev.data_ptr(), g)
              for g in groups]
    s_in, s_cmp, s_out = (torch.cuda.Stream(dev) for _ in range(3))

    def rng(off, sizes, g):
        lo = off[g[0]]
        hi = off[g[-1]] + sizes(g[-1])
        return lo, hi

    def e2e_step():
        main = torch.cuda.current_stream(dev)
        go = torch.cuda.Event()
        go.record(main)
        done = []
        for gi, g in enumerate(groups):
            torch.cuda.nvtx.range_push(f"e2e layer {gi}")
            xl, xh = rng(lay.x_off, lambda i: specs[i].numel_storage * specs[i].elem_bytes, g)
            yl, yh = rng(lay.y_off, lambda i: specs[i].numel, g)
            sl, shh = rng(lay.s_off, lambda i: specs[i].nblocks * 4, g)
            s_in.wait_event(go)
            with torch.cuda.stream(s_in):
                x_dev[xl:xh].copy_(host_t[xl:xh], non_blocking=True)
                e_in = torch.cuda.Event()
                e_in.record(s_in)
            s_cmp.wait_event(e_in)
            st = L.fp8bq_quantize_batched(tables[gi], len(tables[gi]),
                                          ctypes.c_void_p(s_cmp.cuda_stream))
            if st != 0:
                raise RuntimeError(fq.fp8bq_status_string(st))
            e_c = torch.cuda.Event()
            e_c.record(s_cmp)
            s_out.wait_event(e_c)
            with torch.cuda.stream(s_out):
                y_host[yl:yh].copy_(y_dev[yl:yh], non_blocking=True)
                s_host[sl:shh].copy_(s_dev[sl:shh], non_blocking=True)
                e_o = torch.cuda.Event()
                e_o.record(s_out)
            done.append(e_o)
            torch.cuda.nvtx.range_pop()
        for e in done:
            main.wait_event(e)

    e2e_steps = max(1, min(args.steps, args.e2e_steps))
    e2e_step()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    torch.cuda.synchronize()
    e0.record()
    for _ in range(e2e_steps):
        e2e_step()
    e1.record()
    torch.cuda.synchronize()
    dist.barrier()
    fq.check(fq.fp8bq_sync_status(), "e2e steps")
    e2e_elapsed = dist.max(e0.elapsed_time(e1) / 1e3)
    e2e_value = aggregate(bytes_per_step, e2e_steps, world, e2e_elapsed)
    h2d = sum(sp.numel_storage * sp.elem_bytes for sp in specs)
    d2h = sum(sp.numel + sp.nblocks * 4 for sp in specs)

    cpu = None
    if rank == 0 and world == 1 and args.cpu_seconds > 0:
        cpu = cpu_baseline(specs, host, lay, args.cpu_seconds)

    peak, peak_kind = measured_peak()
    l2_mb = torch.cuda.get_device_properties(dev).L2_cache_size / 1e6
    launch_s = elapsed_s / args.steps / max(launches, 1)
    achieved = bytes_per_step / max(launches, 1) / launch_s / 1e9
    # the records are of the grouped call (one call per step); other modes run
    # other launches, so they report no traffic
    traffic, traffic_source = traffic_for(args.workload, args.path, launches) \
        if args.mode == "grouped" and args.repeat == 1 else (None, None)

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": max_elapsed / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wl_desc, "name": args.workload, "tensors": len(specs),
                       "elements": elements, "bytes_per_step": bytes_per_step,
                       "block": list(specs[0].block), "input_dtype": specs[0].dtype, "output_dtype": "e4m3fn",
                       "path": args.path, "calls_per_step": args.mode,
                       "programmatic_dependent_launch": args.pdl,
                       "parallelism": f"replicas x{world}",
                       "l2": (f"no flush: {lay.x_bytes / 1e6:.0f} MB of inputs per step vs "
                              f"{l2_mb:.0f} MB L2") if lay.x_bytes > 2 * l2_mb * 1e6
                       else "inputs fit in L2: latency-bound case",
                       "pct_hbm_peak": value / world / peak * 100.0,
                       "elements_per_s": elements * args.steps * world / max_elapsed},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "traffic_source": traffic_source,
                         "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)"
                         if peak_kind == "measured" else "fallback 6650 GB/s",
                         "kernel_launches_per_step": launches,
                         "avg_launch_ms": launch_s * 1e3},
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps, "pinned_input": pinned_in,
                    "ms_per_step": e2e_elapsed / e2e_steps * 1e3},
            "gpu_launches": launches * args.steps,
            "clocks": clk.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)

    fq.fp8bq_set_path(fq.FP8BQ_PATH_AUTO)
    if pinned_in:
        cudart.cudaHostUnregister(hptr)
    del host_t, host
    dist.barrier()
    if local_rank == 0 and not args.keep_inputs:
        for p in (shm_path, shm_path + ".done"):
            try:
                os.remove(p)
            except OSError:
                pass
    dist.close()


def run_dequant_op(args, specs, lay, y_dev, s_dev, dev, dist, world, rank, wl_desc) -> None:
    """Time fp8bq_dequantize_batched (bf16 output, or fp32 with --dq-out f32)
    over every quantized tensor of the workload, one grouped call per step;
    the codes come from the quantize steps already run."""
    import torch
    import blockwise_fp8_weight_b200 as fq
    oes = 4 if args.dq_out == "f32" else 2
    out_off, o = [], 0
    for sp in specs:
        out_off.append(o)
        o = align(o + sp.numel * oes, 256)
    out = torch.empty(o, dtype=torch.uint8, device=dev)
    L = fq.lib()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)
    table = (fq.fp8bq_dequant_desc * len(specs))()
    for i, sp in enumerate(specs):
        d = table[i]
        d.y_u8 = y_dev.data_ptr() + lay.y_off[i]
        d.descale_f32 = s_dev.data_ptr() + lay.s_off[i]
        d.out = out.data_ptr() + out_off[i]
        d.batch, d.M, d.N = sp.batch, sp.M, sp.N
        d.ld_out, d.out_batch_stride = sp.N, sp.M * sp.N
        d.dtype_out = fq.FP8BQ_F32 if oes == 4 else fq.FP8BQ_BF16
        d.block_m, d.block_n = sp.block
        d.reserved = 0

    def step():
        st = L.fp8bq_dequantize_batched(table, len(specs), sh)
        if st != 0:
            raise RuntimeError(fq.fp8bq_status_string(st))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        while not t1.query():
            time.sleep(0.0005)
        torch.cuda.synchronize()
    dist.barrier()
    el = dist.max(t0.elapsed_time(t1) / 1e3)
    nbytes = sum(sp.numel * (1 + oes) + sp.nblocks * 4 for sp in specs)
    value = aggregate(nbytes, args.steps, world, el)
    peak, kind = measured_peak()
    dq_launches = -(-len(specs) // 320)  # 320 descriptors per launch
    if rank == 0:
        print(json.dumps({
            "metric": f"blockwise FP8 dequantize GB/s (e4m3 codes + descales in, {args.dq_out} out)",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wl_desc + f" (dequantize its codes to {args.dq_out})",
                       "name": args.workload, "op": "dequantize", "bytes_per_step": nbytes,
                       "launches_per_step": dq_launches, "path": args.path},
            "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak, "unit": "GB/s",
                         "frac": value / world / peak, "traffic": None,
                         "peak_source": kind},
            "gpu_launches": dq_launches * args.steps, "clocks": clk.summary()}),
              flush=True)


def run_shard_op(args, specs, lay, x_dev, dev, dist, world, rank, wl_desc) -> None:
    """Time the weight sync of row-sharded weights two ways, every rank holding
    its block-row shard of every (2-D) weight of the workload:
      ours      one grouped quantize launch writes every shard's codes and
                descales into its slot of the gather buffers, then each
                weight's codes and descales are all-gathered in place;
      baseline  each weight's bf16 shards are all-gathered, then the whole
                weights are quantized (one grouped launch).
    Value: ours, in GB/s of the quantizer's algorithmic bytes of the whole
    weights (the same bytes as the default metric)."""
    import socket

    import torch
    import torch.distributed as tdist
    import blockwise_fp8_weight_b200 as fq
    from blockwise_fp8_weight_b200.shard import ShardedQuantGather, shard_rows
    if not tdist.is_initialized():  # one rank: a one-process NCCL group
        sk = socket.socket()
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
        sk.close()
        tdist.init_process_group("nccl", store=tdist.TCPStore("127.0.0.1", port, 1, True),
                                 rank=0, world_size=1, device_id=dev)
    idx = [i for i, sp in enumerate(specs) if sp.batch == 1 and sp.row_stride == sp.N
           and sp.dtype == "bf16"]
    if not idx:
        raise SystemExit("--op shard needs 2-D bf16 tensors without row padding")
    bm, bn = specs[idx[0]].block
    full = [x_dev[lay.x_off[i]:lay.x_off[i] + specs[i].numel * 2].view(torch.bfloat16)
            .view(specs[i].M, specs[i].N) for i in idx]
    ranges = [shard_rows(specs[i].M, world, bm)[rank] for i in idx]
    shards = [f[lo:hi] for f, (lo, hi) in zip(full, ranges)]
    sqg = ShardedQuantGather([(specs[i].M, specs[i].N) for i in idx], (bm, bn), device=dev)
    # baseline buffers: padded bf16 shards (as FSDP keeps them), the gathered
    # bf16 weights, and the quantized outputs
    rows = [-(-(-(-specs[i].M // bm)) // world) * bm for i in idx]
    pad = [torch.zeros((r, specs[i].N), dtype=torch.bfloat16, device=dev) for r, i in zip(rows, idx)]
    for p_, sh in zip(pad, shards):
        p_[:sh.shape[0]].copy_(sh)
    gathered = [torch.empty((world * r, specs[i].N), dtype=torch.bfloat16, device=dev)
                for r, i in zip(rows, idx)]
    outs = [fq._outputs(g[:specs[i].M], (bm, bn)) for g, i in zip(gathered, idx)]
    base_descs = [fq.make_desc(g[:specs[i].M], y, s_, (bm, bn))
                  for g, i, (y, s_) in zip(gathered, idx, outs)]
    base_table = (fq.fp8bq_desc * len(base_descs))(*base_descs)
    L = fq.lib()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)

    def step_ours():
        sqg.run(shards)

    from blockwise_fp8_weight_b200.shard import _coalesced

    def step_base():
        with _coalesced(None, dev):   # the same coalescing of the gathers as ours
            for g, p_ in zip(gathered, pad):
                tdist.all_gather_into_tensor(g.view(torch.uint8), p_.view(torch.uint8))
        st = L.fp8bq_quantize_batched(base_table, len(base_descs), sh)
        if st != 0:
            raise RuntimeError(fq.fp8bq_status_string(st))

    def timed(step):
        for _ in range(args.warmup):
            step()
        torch.cuda.synchronize()
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        dist.barrier()
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        torch.cuda.synchronize()
        dist.barrier()
        return dist.max(t0.elapsed_time(t1) / 1e3)

    with ClockSampler(dev) as clk:
        el_ours = timed(step_ours)
        el_base = timed(step_base)
    # both ways give the same bytes
    res = sqg.run(shards)
    torch.cuda.synchronize()
    same = all(torch.equal(a.view(torch.uint8), y.view(torch.uint8)) and torch.equal(b, s_)
               for (a, b), (y, s_) in zip(res, outs))
    nbytes = sum(specs[i].algorithmic_bytes for i in idx)
    value = aggregate(nbytes, args.steps, world, el_ours)
    peak, kind = measured_peak()
    if rank == 0:
        print(json.dumps({
            "metric": "sharded weight sync: quantize shards + all-gather e4m3 codes, GB/s of "
                      "quantizer bytes of the whole weights",
            "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": el_ours / args.steps * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": {"workload": wl_desc + f"; {len(idx)} weights row-sharded over {world} "
                                             f"rank(s) in whole block rows", "name": args.workload,
                       "op": "shard", "bytes_per_step": nbytes,
                       "gathered_bytes_per_rank_ours": sum(b.codes.numel() + b.descale.numel() * 4
                                                           for b in sqg.bufs),
                       "gathered_bytes_per_rank_baseline": sum(g.numel() * 2 for g in gathered)},
            "baseline_gather_bf16_then_quantize": {
                "value": aggregate(nbytes, args.steps, world, el_base), "unit": "GB/s",
                "ms_per_step": el_base / args.steps * 1e3},
            "same_bytes_both_ways": same,
            "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak, "unit": "GB/s",
                         "frac": value / world / peak, "traffic": None, "peak_source": kind},
            "gpu_launches": None, "clocks": clk.summary()}), flush=True)
    if world == 1:
        tdist.destroy_process_group()


def run_scale_op(args, specs, lay, x_dev, dev, dist, world, rank, wl_desc) -> None:
    """Time fp8bq_tensor_scale over every tensor of the workload (one grouped
    call per step): a read-only pass, numel * elem_bytes + 4 bytes per tensor."""
    import torch
    import blockwise_fp8_weight_b200 as fq
    table = (fq.fp8bq_scale_desc * len(specs))()
    for i, sp in enumerate(specs):
        table[i].x = x_dev.data_ptr() + lay.x_off[i]
        table[i].numel = sp.numel_storage
        table[i].dtype_in = fq.FP8BQ_BF16 if sp.dtype == "bf16" else fq.FP8BQ_F32
        table[i].reserved = 0
    out = torch.empty(len(specs), dtype=torch.float32, device=dev)
    L = fq.lib()
    stream = torch.cuda.current_stream(dev)
    sh = ctypes.c_void_p(stream.cuda_stream)

    def step():
        st = L.fp8bq_tensor_scale(table, len(specs), ctypes.c_void_p(out.data_ptr()), sh)
        if st != 0:
            raise RuntimeError(fq.fp8bq_status_string(st))

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    dist.barrier()
    with ClockSampler(dev) as clk:
        t0.record(stream)
        for _ in range(args.steps):
            step()
        t1.record(stream)
        while not t1.query():
            time.sleep(0.0005)
        torch.cuda.synchronize()
    dist.barrier()
    el = dist.max(t0.elapsed_time(t1) / 1e3)
    nbytes = sum(sp.numel_storage * sp.elem_bytes + 4 for sp in specs)
    value = aggregate(nbytes, args.steps, world, el)
    peak, kind = measured_peak()
    if rank == 0:
        print(json.dumps({
            "metric": "per-tensor FP8 scale GB/s (bytes read)", "value": value, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": el / args.steps * 1e3, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": wl_desc, "name": args.workload, "op": "tensor_scale",
                       "bytes_per_step": nbytes, "tensors": len(specs)},
            "roofline": {"bound": "hbm", "achieved": value / world, "peak": peak, "unit": "GB/s",
                         "frac": value / world / peak, "traffic": None, "peak_source": kind,
                         "note": "one zeroing, one grid-wide pass and one finalize launch per step"},
            "gpu_launches": 3 * args.steps, "clocks": clk.summary()}), flush=True)


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawTextHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="qwen3_8b_model",
                    help="qwen3_8b_model (default), qwen3_8b_layer, qwen3_8b_layer_f32, "
                         "moe_layer, small, act_1x128, blk_64x64, qkv, ragged, edge, or "
                         "shape:[BATCHx]MxN[:f32] for one tensor of that shape")
    ap.add_argument("--path", choices=list(PATHS), default="auto")
    ap.add_argument("--e2e-steps", type=int, default=3)
    ap.add_argument("--repeat", type=int, default=1,
                    help="replicate the workload's tensor list this many times (distinct values)")
    ap.add_argument("--only", default=None, metavar="REGEX",
                    help="keep only the workload's tensors whose name matches REGEX")
    ap.add_argument("--pdl", choices=["on", "off"], default="on",
                    help="programmatic dependent launch of the library's kernels")
    ap.add_argument("--mode", choices=["grouped", "per_layer", "per_tensor"], default="grouped",
                    help="C-ABI calls per step: one grouped call, one per layer, or one per "
                         "tensor")
    ap.add_argument("--dq-out", choices=["bf16", "f32"], default="bf16",
                    help="output dtype of --op dequantize")
    ap.add_argument("--op", choices=["quantize", "dequantize", "tensor_scale", "shard"],
                    default="quantize",
                    help="dequantize: time the reverse map on the quantized workload; "
                         "tensor_scale: time per-tensor scales of the workload's tensors; "
                         "shard: time quantize-then-gather of row-sharded weights against "
                         "gather-then-quantize")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="CPU time spent on the oracle baseline (0 = skip)")
    ap.add_argument("--keep-inputs", action="store_true",
                    help="keep the generated host inputs in /dev/shm for the next run")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")
    _rank, _local, world = dist_env()
    if world != args.gpus and not (world == 1 and args.gpus == 1):
        if world == 1 and args.gpus > 1:
            raise SystemExit("--gpus N > 1 needs torchrun with N processes")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
