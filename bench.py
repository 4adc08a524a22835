"""Benchmark: whole-stack decode throughput of libwcodec on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl {wcodec,reference}]

Workload: the 8B-shaped stack -- 32 Llama-3-8B-shaped decoder layers (q, k,
v, o, gate, up, down) plus embedding and LM head, 226 BF16 tensors,
8,029,995,008 elements (16.06 GB), Gaussian N(0, 0.02) with a per-matrix std
jitter of +/-30%, drawn on the GPU from fixed seeds -- at block size B=1024.

A step runs the whole hot path once: compress all 226 tensors (split, width,
scan, pack: one batched encoder launch) and decompress all of them (one
batched decoder launch). Both phases are timed with CUDA events on the
launching stream; the metric is the decode phase: BF16 bytes produced per
second (2 bytes per element). Inputs (16 GB per pass) are far larger than the
126 MB L2, so no flush is needed between steps.

One JSON line goes to stdout (rank 0). ``--impl reference`` times the CPU
oracle instead, on a bounded sample of the same workload, on the host cores.
Under torchrun every rank draws its own stack (weak scaling, no data-path
collective); times are the maximum over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode GB/s (BF16 out) & % HBM roofline at 1 B200; compression ratio"
BLOCK = 1024
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0
WORKLOAD = ("llama3_8b_stack: 32 Llama-3-8B-shaped decoder layers + embedding + LM head "
            "(226 BF16 tensors, 8,029,995,008 elements, 16.06 GB), N(0, 0.02) with per-matrix "
            "std jitter U[0.7, 1.3], block 1024")
LAYER_WORKLOAD = ("llama3_8b_layer: one Llama-3-8B-shaped decoder layer (7 BF16 tensors, "
                  "218,103,808 elements, 436 MB), block 1024 -- a smaller case for profiling")


def log(*a):
    print(*a, file=sys.stderr, flush=True)


# ---------------------------------------------------------------------------
# distributed plumbing (one process per GPU; NCCL only for timing reductions)
# ---------------------------------------------------------------------------
def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def init_dist(world, backend):
    import datetime

    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=300))
    return dist if world > 1 else None


def max_over_ranks(value: float, dist, device) -> float:
    import torch
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(dist, device):
    import torch
    if dist is not None:
        if device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()
    if device.type == "cuda":
        torch.cuda.synchronize(device)


def whole_job_gbs(world: int, bytes_per_rank: float, steps: int, max_seconds: float) -> float:
    """Whole-job throughput: the bytes all ranks produced over the slowest rank's time."""
    return world * bytes_per_rank * steps / max_seconds / 1e9


def rank_seed_base(rank: int) -> int:
    """Seeds of rank r's stack: every rank draws a different, fixed stack."""
    return 10 + 100_000 * rank


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
CLOCK_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
                "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
                "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


class ClockSampler:
    def __init__(self, gpu_index: int):
        self.path = tempfile.mktemp(prefix="wc_clocks_", suffix=".csv")
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + CLOCK_FIELDS,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        reasons = sorted({names[k] for r in rows for k, v in enumerate(r[3]) if v == "Active"})
        loaded = [r[0] for r in rows if r[2] > 200.0] or [r[0] for r in rows]
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": max(r[1] for r in rows),
                "power_w_max": max(r[2] for r in rows), "samples": len(rows), "reasons": reasons}


# ---------------------------------------------------------------------------
# roofline denominators and ncu traffic
# ---------------------------------------------------------------------------
def hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback"


def decode_kernel_digest() -> str:
    h = hashlib.sha256()
    for name in ("wc_decode.cu", "wc_decode_core.cuh", "wc_internal.cuh"):
        with open(os.path.join(ROOT, "lossless_weight_compression_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def ncu_traffic_per_elem():
    """DRAM bytes per element of one decode launch, from the committed ncu
    summary (dram__bytes_read.sum + dram__bytes_write.sum of one launch over
    ``elements`` elements), or None if there is none or the decoder's source
    changed since the counters were taken."""
    path = os.path.join(ROOT, "profiles", "decode_kernel_traffic.txt")
    try:
        fields = dict(line.split(":", 1) for line in open(path) if ":" in line)
    except OSError:
        return None
    fields = {k.strip(): v.strip() for k, v in fields.items()}
    if fields.get("kernel_source_digest") != decode_kernel_digest():
        return None
    try:
        return float(fields["dram_bytes_per_launch"]) / float(fields["elements"])
    except (KeyError, ValueError, ZeroDivisionError):
        return None


# ---------------------------------------------------------------------------
# the CPU oracle, timed (cpu_baseline and the reference arm)
# ---------------------------------------------------------------------------
def host_info():
    """The host the oracle runs on: its usable core count and CPU model."""
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"host_cores": cores, "cpu_model": model}


ORACLE_SAMPLE = ("layer 0 of the stack (7 tensors, 218,103,808 elements) copied to the host; "
                 "the single-threaded C oracle encodes each tensor once (timed apart), then "
                 "decodes all seven per step (the metric)")


def oracle_sample_words(device_tensors=None):
    """The bounded sample the oracle is timed on, in both the cpu_baseline and the
    reference arm: layer 0 of the stack (7 tensors, 218,103,808 elements), as
    host uint16 arrays."""
    import numpy as np
    import torch

    from lossless_weight_compression_b200 import synth
    out = []
    if device_tensors is not None:
        for name, t in device_tensors:
            if name.startswith("layers.0."):
                out.append((name, t.view(-1).view(torch.int16).cpu().numpy().view(np.uint16)))
    else:
        for name, t in synth.layer_tensors(0, "cpu", rank_seed_base(0)):
            out.append((name, t.view(-1).view(torch.int16).numpy().view(np.uint16)))
    return out


class OracleTimer:
    """The oracle on a host sample: encode() once, then decode_step() per step."""

    def __init__(self, sample, block=BLOCK):
        import oracle
        oracle.build()
        self.oracle, self.sample, self.block = oracle, sample, block
        self.n = sum(w.size for _, w in sample)
        self.streams = None

    def encode(self):
        """Encode every tensor once; returns BF16-in GB/s."""
        t0 = time.perf_counter()
        self.streams = [self.oracle.compress(w, self.block) for _, w in self.sample]
        return 2 * self.n / (time.perf_counter() - t0) / 1e9

    def decode_step(self):
        """Decode every tensor once and check it; returns the seconds spent decoding."""
        import numpy as np
        sec = 0.0
        for (_, w), s in zip(self.sample, self.streams):
            t0 = time.perf_counter()
            d = self.oracle.decompress(s, w.size, self.block)
            sec += time.perf_counter() - t0
            if not np.array_equal(d, w):
                raise RuntimeError("oracle round trip failed")
        return sec


def run_reference(args):
    world, rank, _ = dist_env()
    if rank != 0:
        return 0
    import torch
    torch.set_num_threads(1)
    timer = OracleTimer(oracle_sample_words())
    enc_gbs = timer.encode()
    for _ in range(args.warmup):
        timer.decode_step()
    total = sum(timer.decode_step() for _ in range(args.steps))
    value = 2 * timer.n * args.steps / total / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": WORKLOAD, "block": BLOCK,
                   "sample": "per step: " + ORACLE_SAMPLE},
        "cpu_baseline": dict({"value": value, "unit": "GB/s", "cores": 1, "kind": "oracle",
                              "sample": ORACLE_SAMPLE, "encode_gbs_bf16_in": enc_gbs},
                             **host_info()),
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the GPU arm
# ---------------------------------------------------------------------------
def timed_steps(fn, steps, warmup, stream, dist, dev):
    """Seconds per call of fn: `warmup` untimed calls, then `steps` calls between
    two CUDA events on `stream`, barriers on both sides, max over ranks."""
    import torch
    for _ in range(warmup):
        fn()
    barrier(dist, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        fn()
    e1.record(stream)
    barrier(dist, dev)
    return max_over_ranks(e0.elapsed_time(e1) / 1e3 / steps, dist, dev)


def escape_phase(args, wc, wcodec, inputs, outs, stream, dist, dev, world, mats=None):
    """The same tensors as escape-coded streams: one wc_compress_escape_batch call
    (five launches) and one wc_decompress_escape_batch launch, each timed over
    the step count; every decoded tensor checked against its input. mats:
    (index, (rows, cols) BF16 view) of the linear weights, multiplied from
    their escape-coded streams on the tensor cores at args.fused_tokens."""
    import torch
    sh = stream.cuda_stream
    n_total = sum(w.numel() for w in inputs)
    enc = wcodec.CompressBatch(inputs, block=BLOCK, escape=True)
    status = torch.zeros(2, dtype=torch.int32, device=dev)

    def encode_all():
        rc = wc.wc_compress_escape_batch(enc.items, enc.count, enc.workspace.data_ptr(),
                                         enc.workspace.numel(), status[0:].data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_compress_escape_batch: %s" % wc.wc_status_string(rc))

    encode_all()
    torch.cuda.synchronize(dev)
    sizes = enc.sizes()
    batch = wcodec.make_batch([(enc.buffers[k], sizes[k], outs[k], inputs[k].numel(), BLOCK)
                               for k in range(len(inputs))])

    def decode_all():
        rc = wc.wc_decompress_escape_batch(batch[0], batch[1], status[1:].data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_decompress_escape_batch: %s" % wc.wc_status_string(rc))

    for o in outs:
        o.fill_(-1)
    torch.cuda.nvtx.range_push("escape-coded encode")
    t_enc = timed_steps(encode_all, args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.nvtx.range_push("escape-coded decode")
    t_dec = timed_steps(decode_all, args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    ok = (bool((status == 0).all().item()) and enc.sizes() == sizes
          and all(torch.equal(a, b) for a, b in zip(inputs, outs)))
    C = sum(sizes)
    moved = C + 2 * n_total
    peak, peak_kind = hbm_peak()
    out = {"value": world * 2 * n_total / t_dec / 1e9, "unit": "GB/s (BF16 out)",
           "ms_per_step": 1e3 * t_dec,
           "roofline": {"bound": "hbm", "achieved": moved / t_dec / 1e9, "peak": peak,
                        "unit": "GB/s", "frac": moved / t_dec / 1e9 / peak,
                        "peak_kind": peak_kind,
                        "kernel": "decode_kernel<512,escape> (one launch per step)",
                        "algorithmic_bytes_per_launch": moved},
           "compression": {"ratio": 2 * n_total / C, "stream_bytes": C},
           "encode": {"ms_per_step": 1e3 * t_enc, "achieved_hbm_gbs": moved / t_enc / 1e9,
                      "frac_of_peak": moved / t_enc / 1e9 / peak,
                      "kernels": "esc_params, esc_reduce, esc_top, esc_down, esc_pack (one "
                                 "launch each per step)"},
           "gpu_launches": args.steps * 6,
           "verified_bit_exact": ok}
    fused = []
    for nv in (args.fused_tokens if mats else []):
        res, fok = fused_phase(args, wc, wcodec, [m for _, m in mats],
                               [enc.buffers[k] for k, _ in mats], [sizes[k] for k, _ in mats],
                               nv, True, stream, dist, dev, world, escape=True)
        fused.append(res)
        ok &= fok
    out["fused_gemm"] = fused or None
    out["verified_bit_exact"] = ok
    del enc, batch
    torch.cuda.empty_cache()
    return out, ok


TANS_CHUNK = 4096
TANS_LOG = 10


def tans_phase(args, wc, wcodec, inputs, outs, stream, dist, dev, world):
    """The same tensors as tANS-coded streams (exponents entropy-coded, chunks
    of 4096 elements as 32 interleaved lane streams, 2^10 states): one
    wc_compress_tans_batch call (five launches) and one wc_decompress_tans_batch
    launch, each timed over the step count; every decoded tensor checked
    against its input."""
    import torch
    n_total = sum(w.numel() for w in inputs)
    enc = wcodec.CompressBatch(inputs, block=TANS_CHUNK, tans_log=TANS_LOG)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    enc.run(stream)
    torch.cuda.synchronize(dev)
    sizes = enc.sizes()
    batch = wcodec.make_batch([(enc.buffers[k], sizes[k], outs[k], inputs[k].numel(), TANS_CHUNK)
                               for k in range(len(inputs))])

    def decode_all():
        wcodec.decompress_tans_batch(batch, status, stream)

    for o in outs:
        o.fill_(-1)
    torch.cuda.nvtx.range_push("tANS encode")
    t_enc = timed_steps(lambda: enc.run(stream), args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.nvtx.range_push("tANS decode")
    t_dec = timed_steps(decode_all, args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    ok = (status.item() == 0 and enc.sizes() == sizes
          and all(torch.equal(a, b) for a, b in zip(inputs, outs)))
    C = sum(sizes)
    moved = C + 2 * n_total
    peak, peak_kind = hbm_peak()
    out = {"value": world * 2 * n_total / t_dec / 1e9, "unit": "GB/s (BF16 out)",
           "ms_per_step": 1e3 * t_dec, "chunk": TANS_CHUNK, "table_log": TANS_LOG,
           "roofline": {"bound": "hbm", "achieved": moved / t_dec / 1e9, "peak": peak,
                        "unit": "GB/s", "frac": moved / t_dec / 1e9 / peak,
                        "peak_kind": peak_kind,
                        "kernel": "tans_decode_kernel<256> (one launch per step)",
                        "algorithmic_bytes_per_launch": moved},
           "compression": {"ratio": 2 * n_total / C, "stream_bytes": C},
           "encode": {"ms_per_step": 1e3 * t_enc, "achieved_hbm_gbs": moved / t_enc / 1e9,
                      "frac_of_peak": moved / t_enc / 1e9 / peak,
                      "kernels": "tans_hist, tans_plan, tans_encode (twice), tans_scan (five "
                                 "launches per step)"},
           "gpu_launches": args.steps * 6,
           "verified_bit_exact": bool(ok)}
    del enc, batch
    torch.cuda.empty_cache()
    return out, bool(ok)


def fused_phase(args, wc, wcodec, mats, streams, sizes, nv, gemm, stream, dist, dev, world,
                escape=False):
    """Fused decode + products over weight matrices given as streams: one
    wc_gemm_batch call (tensor cores, `nv` activation rows, one launch per 64
    matrices) or one wc_gemv_batch launch (`nv` vectors), against torch's BF16
    matmul (cuBLAS) on the uncompressed matrices replayed from a CUDA graph.
    mats: (rows, cols) BF16 tensors; streams/sizes: their streams. Every output
    is checked against the float64 product of the uncompressed weights."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(7)
    xs = [torch.randn((nv, t.shape[1]), generator=g, device=dev).to(torch.bfloat16) for t in mats]
    ys = [torch.empty((nv, t.shape[0]), dtype=torch.float32, device=dev) for t in mats]
    batch = wcodec.make_gemv_batch([(streams[k], sizes[k], xs[k], ys[k], t.shape[0], t.shape[1],
                                     BLOCK) for k, t in enumerate(mats)])
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    if gemm:
        entry, ename = (wc.wc_gemm_batch, "wc_gemm_batch")
    else:
        entry, ename = (wc.wc_gemv_batch, "wc_gemv_batch")
    flags = 2 if escape else 0

    def fused():
        if flags:
            rc = wc.wc_gemm_batch_flags(batch[0], batch[1], nv, flags, status.data_ptr(),
                                        stream.cuda_stream)
        else:
            rc = entry(batch[0], batch[1], nv, status.data_ptr(), stream.cuda_stream)
        if rc != 0:
            raise RuntimeError("%s: %s" % (ename, wc.wc_status_string(rc)))

    outs = [torch.empty((nv, t.shape[0]), dtype=torch.bfloat16, device=dev) for t in mats]
    side = torch.cuda.Stream(dev)
    side.wait_stream(stream)
    with torch.cuda.stream(side):
        for _ in range(2):
            for k, t in enumerate(mats):
                torch.matmul(xs[k], t.T, out=outs[k])
    stream.wait_stream(side)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for k, t in enumerate(mats):
            torch.matmul(xs[k], t.T, out=outs[k])
    what = "gemm" if gemm else "gemv"
    torch.cuda.nvtx.range_push("fused decode+%s, %d rows" % (what, nv))
    t_fused = timed_steps(fused, args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.nvtx.range_push("cuBLAS BF16, %d rows" % nv)
    t_blas = timed_steps(graph.replay, args.steps, args.warmup, stream, dist, dev)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    ok = status.item() == 0
    for k, t in enumerate(mats):
        ref = xs[k].double() @ t.double().T
        # FP32 sum bound; the tensor cores' accumulation is held to 4x that
        scale = t.shape[1] * 2.0 ** -22 if gemm else (t.shape[1] - 1) * 2.0 ** -24
        bound = scale * (xs[k].double().abs() @ t.double().abs().T)
        ok &= bool(((ys[k].double() - ref).abs() <= bound).all())
        del ref, bound
    weights = sum(t.numel() for t in mats)
    stream_bytes = sum(sizes)
    x_bytes = sum(x.numel() * 2 for x in xs)
    y_bytes = sum(y.numel() * 4 for y in ys)
    moved = stream_bytes + x_bytes + y_bytes
    peak, peak_kind = hbm_peak()
    launches = -(-len(mats) // 64) if gemm else -(-len(mats) // 256)
    kernel = ("gemm_kernel<64%s> (tcgen05, %d launches per step)"
              % (",escape" if escape else "", launches) if gemm
              else "gemv_kernel<256,%d> (%d launches per step)" % (nv, launches))
    out = {"tokens" if gemm else "n_vec": nv,
           "value": world * 2 * weights / t_fused / 1e9, "unit": "GB/s (effective BF16 weights)",
           "ms_per_step": 1e3 * t_fused,
           "roofline": {"bound": "hbm", "achieved": moved / t_fused / 1e9, "peak": peak,
                        "unit": "GB/s", "frac": moved / t_fused / 1e9 / peak,
                        "peak_kind": peak_kind, "kernel": kernel,
                        "algorithmic_bytes_per_launch": moved / launches},
           "cublas_bf16": {"ms_per_step": 1e3 * t_blas,
                           "achieved_gbs": (2 * weights + x_bytes + 2 * sum(o.numel() for o in outs))
                           / t_blas / 1e9,
                           "speedup_of_fused": t_blas / t_fused},
           "tflops": 2.0 * weights * nv / t_fused / 1e12,
           "stream": "escape-coded" if escape else "plain",
           "gpu_launches": args.steps * launches,
           "verified_within_fp32_bound": bool(ok)}
    del graph, xs, ys, outs
    torch.cuda.empty_cache()
    return out, bool(ok)


def run_wcodec(args):
    import torch

    from lossless_weight_compression_b200 import build_lib, synth, wcodec

    world, rank, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (B200)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    build_lib.build()
    wc = wcodec.lib()
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream

    # ---- workload, resident in HBM ------------------------------------------------
    t0 = time.time()
    names, inputs, shapes = [], [], []
    hist = torch.zeros(256, dtype=torch.int64, device=dev)
    if args.workload == "stack":
        tensors = synth.stack_tensors(dev, rank_seed_base(rank))
    else:
        tensors = synth.layer_tensors(0, dev, rank_seed_base(rank))
    for name, t in tensors:
        words = t.view(-1).view(torch.int16)
        hist += torch.bincount(((words.to(torch.int32) >> 7) & 0xFF), minlength=256)
        names.append(name)
        inputs.append(words)
        shapes.append(tuple(t.shape))
    n_total = sum(w.numel() for w in inputs)
    log("rank %d: generated %d tensors, %d elements in %.1f s" % (rank, len(inputs), n_total,
                                                                   time.time() - t0))

    # ---- buffers for every tensor (no allocation inside the timed region) ----------
    enc = wcodec.CompressBatch(inputs, block=BLOCK)
    bufs = enc.buffers
    outs = [torch.empty(w.numel(), dtype=torch.int16, device=dev) for w in inputs]
    status = torch.zeros(2, dtype=torch.int32, device=dev)

    def encode_all():  # one batched encoder launch for all tensors
        rc = wc.wc_compress_batch(enc.items, enc.count, enc.workspace.data_ptr(),
                                  enc.workspace.numel(), status[0:].data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_compress_batch: %s" % wc.wc_status_string(rc))

    encode_all()
    torch.cuda.synchronize(dev)
    sizes = enc.sizes()
    batch = wcodec.make_batch([(bufs[k], sizes[k], outs[k], inputs[k].numel(), BLOCK)
                               for k in range(len(inputs))])
    dec_status = status[1:]

    def decode_all():
        rc = wc.wc_decompress_batch(batch[0], batch[1], dec_status.data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_decompress_batch: %s" % wc.wc_status_string(rc))

    stream_total = sum(sizes)
    exp_total = 0
    for k in range(len(inputs)):
        header = bufs[k][:128].cpu().numpy().tobytes()
        exp_total += int.from_bytes(header[64:72], "little")

    # ---- warm-up, then K timed steps (encode phase, decode phase) -------------------
    for _ in range(args.warmup):
        encode_all()
        decode_all()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(dist, dev)
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        for k in range(args.steps):
            torch.cuda.nvtx.range_push("encode (A1-A4), step %d" % k)
            ev[k][0].record(stream)
            encode_all()
            ev[k][1].record(stream)
            torch.cuda.nvtx.range_pop()
            torch.cuda.nvtx.range_push("decode (A5), step %d" % k)
            ev[k][2].record(stream)
            decode_all()
            ev[k][3].record(stream)
            torch.cuda.nvtx.range_pop()
        barrier(dist, dev)
    enc_ms = [e[0].elapsed_time(e[1]) for e in ev]
    dec_ms = [e[2].elapsed_time(e[3]) for e in ev]
    dec_total_s = max_over_ranks(sum(dec_ms) / 1e3, dist, dev)
    enc_total_s = max_over_ranks(sum(enc_ms) / 1e3, dist, dev)

    # ---- verification (outside the timed region) -----------------------------------
    torch.cuda.synchronize(dev)
    verified = bool((status == 0).all().item()) and all(
        torch.equal(a, b) for a, b in zip(inputs, outs))
    verified &= enc.sizes() == sizes

    # ---- end to end: compressed streams from pinned host memory ---------------------
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wc, wcodec, bufs, sizes, batch, dec_status, inputs, outs, stream, dist,
                      dev, n_total)

    # ---- the next rows on the same weights: escape-coded streams, fused products --------
    extra_ok = True
    # the linear weights (the embedding is a lookup, not a product)
    idx = [k for k, nm in enumerate(names) if nm != "embed_tokens"]
    mats = [inputs[k].view(torch.bfloat16).view(shapes[k]) for k in idx]
    escape = None
    if not args.no_escape:
        escape, ok = escape_phase(args, wc, wcodec, inputs, outs, stream, dist, dev, world,
                                  list(zip(idx, mats)))
        extra_ok &= ok
    tans = None
    if not args.no_tans:
        tans, ok = tans_phase(args, wc, wcodec, inputs, outs, stream, dist, dev, world)
        extra_ok &= ok
    fused = []
    if args.fused_tokens:
        # from the plain streams the main encoder wrote
        for nv in args.fused_tokens:
            res, ok = fused_phase(args, wc, wcodec, mats, [bufs[k] for k in idx],
                                  [sizes[k] for k in idx], nv, True, stream, dist, dev, world)
            fused.append(res)
            extra_ok &= ok

    # ---- figures ---------------------------------------------------------------------
    bytes_out = 2 * n_total
    value = whole_job_gbs(world, bytes_out, args.steps, dec_total_s)
    moved = stream_total + bytes_out  # algorithmic bytes of one decode launch: read C, write 2n
    dec_launch_s = dec_total_s / args.steps
    achieved = moved / dec_launch_s / 1e9
    peak, peak_kind = hbm_peak()
    traffic_per_elem = ncu_traffic_per_elem()
    p = hist.double() / hist.sum()
    H = float(-(p[p > 0] * torch.log2(p[p > 0])).sum())
    ratio = bytes_out / stream_total
    rho_fmt = bytes_out / (exp_total + n_total)
    clk = clocks.summary()

    line = None
    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            timer = OracleTimer(oracle_sample_words(list(zip(names, inputs))))
            cenc = timer.encode()
            reps = 3
            csec = sum(timer.decode_step() for _ in range(reps))
            cpu = dict({"value": 2 * timer.n * reps / csec / 1e9, "unit": "GB/s", "cores": 1,
                        "kind": "oracle", "sample": ORACLE_SAMPLE + "; %d steps" % reps,
                        "encode_gbs_bf16_in": cenc}, **host_info())
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * dec_launch_s, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "u16", "data": "synthetic",
            "config": {"workload": WORKLOAD if args.workload == "stack" else LAYER_WORKLOAD,
                       "block": BLOCK, "tensors": len(inputs),
                       "elements_per_gpu": n_total, "parallelism": "replicas: one stack per GPU",
                       "l2": "inputs larger than L2 (%.2f GB BF16 in, %.2f GB stream per pass "
                             "vs 126 MB L2); no flush" % (bytes_out / 1e9, stream_total / 1e9),
                       "step": "compress all %d tensors (1 batched encoder launch) + decompress "
                               "all (1 batched decoder launch); value times the decode phase"
                               % len(inputs)},
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "peak_kind": peak_kind,
                         "frac_of_nominal_8000": achieved / NOMINAL_HBM_GBS,
                         "kernel": "decode_kernel<512> (one launch per step)",
                         "algorithmic_bytes_per_launch": moved,
                         "traffic": (traffic_per_elem * n_total) if traffic_per_elem else None},
            "compression": {"ratio": ratio, "stream_bytes": stream_total,
                            "exponent_entropy_bits": H, "entropy_bound_ratio": 16.0 / (8.0 + H),
                            "format_payload_bound_ratio": rho_fmt,
                            "ratio_over_format_bound": ratio / rho_fmt},
            "encode": {"value": whole_job_gbs(world, bytes_out, args.steps, enc_total_s),
                       "unit": "GB/s (BF16 in)", "kernel": "encode_kernel<512> (one launch per step)",
                       "ms_per_step": 1e3 * enc_total_s / args.steps,
                       "achieved_hbm_gbs": (bytes_out + stream_total) / (enc_total_s / args.steps) / 1e9},
            "e2e": e2e,
            "gpu_launches": args.steps * 2,
            "clocks": clk,
            "verified_bit_exact": verified,
            "cpu_baseline": cpu,
            "escape_coded": escape,
            "tans_coded": tans,
            "fused_gemm": fused or None,
        }
    if dist is not None:
        barrier(dist, dev)
        dist.destroy_process_group()
    if line is not None:
        print(json.dumps(line), flush=True)
    return 0 if (verified and extra_ok) else 1


def run_e2e(args, wc, wcodec, bufs, sizes, batch, dec_status, inputs, outs, stream, dist, dev,
            n_total, entry="wc_decompress_batch", host_flags=0):
    """Same metric through the public C-ABI with the compressed streams in pinned
    host memory and a read of the status word back every step, both inside the
    timed region, by two paths: (a) copy the streams to the device
    (cudaMemcpyAsync per tensor), then one batched decode (`entry`); (b) one
    wc_decompress_host_batch launch that reads the streams over the host link
    itself (`host_flags`: the streams' kind). Path (b), the library call alone,
    is the line's value; (a) is reported beside it."""
    import torch
    decode_batch = getattr(wc, entry)
    total = sum(sizes)
    try:
        host = torch.empty(total, dtype=torch.uint8, pin_memory=True)
    except RuntimeError as exc:
        log("e2e: cannot pin %d bytes: %s" % (total, exc))
        return {"value": None, "unit": "GB/s", "h2d_bytes_per_step": total,
                "d2h_bytes_per_step": 4, "error": "pinned host buffer unavailable"}
    views, off = [], 0
    for k, s in enumerate(sizes):
        views.append(host[off:off + s])
        views[-1].copy_(bufs[k][:s])
        off += s
    status_host = torch.zeros(1, dtype=torch.int32, pin_memory=True)
    sh = stream.cuda_stream

    def step():
        for k, s in enumerate(sizes):
            bufs[k][:s].copy_(views[k], non_blocking=True)
        rc = decode_batch(batch[0], batch[1], dec_status.data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("%s: %s" % (entry, wc.wc_status_string(rc)))
        status_host.copy_(dec_status, non_blocking=True)

    steps = max(1, min(args.steps, 5))
    step()
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(steps):
        step()
    e1.record(stream)
    barrier(dist, dev)
    sec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, dev)
    ok = status_host.item() == 0 and all(torch.equal(a, b) for a, b in zip(inputs, outs))
    world = dist.get_world_size() if dist is not None else 1
    copy_path = {"value": whole_job_gbs(world, 2 * n_total, steps, sec), "unit": "GB/s",
                 "h2d_bytes_per_step": total, "d2h_bytes_per_step": 4, "steps": steps,
                 "path": "cudaMemcpyAsync of each stream, then %s" % entry,
                 "verified_bit_exact": bool(ok)}

    # (b) the decoder reads the pinned streams itself
    for o in outs:
        o.fill_(-1)
    hbatch = wcodec.make_batch([(views[k], sizes[k], outs[k], inputs[k].numel(), BLOCK)
                                for k in range(len(sizes))])

    def fused_step():
        rc = wc.wc_decompress_host_batch(hbatch[0], hbatch[1], host_flags, dec_status.data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_decompress_host_batch: %s" % wc.wc_status_string(rc))
        status_host.copy_(dec_status, non_blocking=True)

    fused_step()
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    e0.record(stream)
    for _ in range(steps):
        fused_step()
    e1.record(stream)
    barrier(dist, dev)
    fsec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, dev)
    fok = status_host.item() == 0 and all(torch.equal(a, b) for a, b in zip(inputs, outs))
    fused_path = {"value": whole_job_gbs(world, 2 * n_total, steps, fsec), "unit": "GB/s",
                  "h2d_bytes_per_step": total, "d2h_bytes_per_step": 4, "steps": steps,
                  "path": "wc_decompress_host_batch (the decoder reads the pinned streams)",
                  "verified_bit_exact": bool(fok)}
    # the value: the library's own host-stream entry point, C-ABI end to end; the
    # copy engines' path (torch copies, then the library's device decode) beside it
    result = dict(fused_path)
    result["copy_then_decode"] = copy_path
    del host, views, hbatch
    # context: the same weights moved uncompressed (BF16, pinned host -> device), no decode
    try:
        raw = torch.empty(2 * n_total, dtype=torch.uint8, pin_memory=True)
    except RuntimeError:
        return result
    raw_views, off = [], 0
    for w in inputs:
        nbytes = 2 * w.numel()
        raw_views.append(raw[off:off + nbytes])
        raw_views[-1].copy_(w.view(torch.uint8))
        off += nbytes

    def raw_step():
        for k, w in enumerate(inputs):
            outs[k].view(torch.uint8).copy_(raw_views[k], non_blocking=True)

    raw_step()
    torch.cuda.synchronize(dev)
    barrier(dist, dev)
    e0.record(stream)
    for _ in range(steps):
        raw_step()
    e1.record(stream)
    barrier(dist, dev)
    raw_sec = max_over_ranks(e0.elapsed_time(e1) / 1e3, dist, dev)
    result["bf16_h2d_only"] = {"value": whole_job_gbs(world, 2 * n_total, steps, raw_sec),
                               "unit": "GB/s", "h2d_bytes_per_step": 2 * n_total,
                               "speedup_of_host_stream_decode": raw_sec / fsec,
                               "speedup_of_copy_then_decode": raw_sec / sec}
    return result


# ---------------------------------------------------------------------------
# next row: escape-coded streams of the whole stack
# ---------------------------------------------------------------------------
def run_escape(args):
    """The 8B-shaped stack as escape-coded streams (a window of 2^w - 1
    exponents per block plus an exception list): all tensors encoded by one
    wc_compress_escape_batch call (five launches), then the whole stack decoded
    by one wc_decompress_escape_batch launch per step (the metric)."""
    import numpy as np
    import torch

    import oracle
    from lossless_weight_compression_b200 import build_lib, synth, wcodec

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    build_lib.build()
    wc = wcodec.lib()
    stream = torch.cuda.current_stream(dev)
    sh = stream.cuda_stream
    names, inputs = [], []
    hist = torch.zeros(256, dtype=torch.int64, device=dev)
    tensors = (synth.stack_tensors(dev, rank_seed_base(rank)) if args.workload == "escape"
               else synth.layer_tensors(0, dev, rank_seed_base(rank)))
    for name, t in tensors:
        words = t.view(-1).view(torch.int16)
        hist += torch.bincount(((words.to(torch.int32) >> 7) & 0xFF), minlength=256)
        names.append(name)
        inputs.append(words)
    n_total = sum(w.numel() for w in inputs)
    enc = wcodec.CompressBatch(inputs, block=BLOCK, escape=True)
    bufs, nbytes = enc.buffers, enc.nbytes
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    outs = [torch.empty(w.numel(), dtype=torch.int16, device=dev) for w in inputs]

    def encode_all():  # five launches for the whole batch
        rc = wc.wc_compress_escape_batch(enc.items, enc.count, enc.workspace.data_ptr(),
                                         enc.workspace.numel(), status[0:].data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_compress_escape_batch: %s" % wc.wc_status_string(rc))

    encode_all()
    torch.cuda.synchronize(dev)
    sizes = enc.sizes()
    batch = wcodec.make_batch([(bufs[k], sizes[k], outs[k], inputs[k].numel(), BLOCK)
                               for k in range(len(inputs))])
    dec_status = status[1:]

    def decode_all():
        rc = wc.wc_decompress_escape_batch(batch[0], batch[1], dec_status.data_ptr(), sh)
        if rc != 0:
            raise RuntimeError("wc_decompress_escape_batch: %s" % wc.wc_status_string(rc))

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        barrier(dist, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        barrier(dist, dev)
        return max_over_ranks(e0.elapsed_time(e1) / 1e3 / args.steps, dist, dev)

    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        t_enc = timed(encode_all)
        t_dec = timed(decode_all)
    torch.cuda.synchronize(dev)
    verified = bool((status == 0).all().item()) and all(
        torch.equal(a, b) for a, b in zip(inputs, outs)) and enc.sizes() == sizes
    e2e = None
    if not args.no_e2e:
        e2e = run_e2e(args, wc, wcodec, bufs, sizes, batch, dec_status, inputs, outs, stream, dist,
                      dev, n_total, entry="wc_decompress_escape_batch", host_flags=2)
    stream_total = sum(sizes)
    bytes_out = 2 * n_total
    moved = stream_total + bytes_out
    peak, peak_kind = hbm_peak()
    p = hist.double() / hist.sum()
    H = float(-(p[p > 0] * torch.log2(p[p > 0])).sum())
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        torch.set_num_threads(1)
        q = [w for nm, w in zip(names, inputs) if nm.endswith("q_proj")][0]
        qw = q.cpu().numpy().view(np.uint16)
        oracle.build()
        t0 = time.perf_counter()
        sref = oracle.compress_escape(qw, BLOCK)
        t1 = time.perf_counter()
        back = oracle.decompress_escape(sref, qw.size, BLOCK)
        t2 = time.perf_counter()
        same = bool(np.array_equal(back, qw)) and bool(np.array_equal(
            sref, bufs[names.index([nm for nm in names if nm.endswith("q_proj")][0])]
            [:sref.size].cpu().numpy()))
        cpu = {"value": 2 * qw.size / (t2 - t1) / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
               "sample": "the first q_proj of the workload (%d elements) copied to the host, "
                         "encoded then decoded once by the single-threaded C oracle; decode "
                         "timed (encode %.4f GB/s); oracle stream equals the GPU's: %s"
                         % (qw.size, 2 * qw.size / (t1 - t0) / 1e9, same)}
        verified &= same
    line = {
        "metric": "escape-coded decode GB/s (BF16 out) & % HBM roofline; compression ratio",
        "value": world * bytes_out / t_dec / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_dec, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": (WORKLOAD if args.workload == "escape" else LAYER_WORKLOAD)
                   + "; escape-coded streams", "block": BLOCK, "tensors": len(inputs),
                   "l2": "inputs larger than L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": moved / t_dec / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": moved / t_dec / 1e9 / peak, "peak_kind": peak_kind,
                     "kernel": "decode_kernel<512,escape> (one launch per step)",
                     "algorithmic_bytes_per_launch": moved, "traffic": None},
        "compression": {"ratio": bytes_out / stream_total, "stream_bytes": stream_total,
                        "exponent_entropy_bits": H, "entropy_bound_ratio": 16.0 / (8.0 + H)},
        "encode": {"ms_per_step": 1e3 * t_enc, "gbs_moved": moved / t_enc / 1e9,
                   "frac_of_peak": moved / t_enc / 1e9 / peak,
                   "kernels": "esc_params, esc_reduce, esc_top, esc_down, esc_pack (one launch "
                              "each for the batch)"},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks.summary(),
        "verified_bit_exact": verified,
        "cpu_baseline": cpu,
    }
    if dist is not None:
        barrier(dist, dev)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if verified else 1


# ---------------------------------------------------------------------------
# every workload at every block size it names, both stream kinds
# ---------------------------------------------------------------------------
def run_sweep(args):
    """Encode and decode timings of workloads 1, 2, 3 and 5 at each of their block
    sizes, as plain and as escape-coded streams (one batched launch per
    direction; workload 4 is the default benchmark). A case whose input, stream
    and output together fit in the 126 MB L2 is flagged L2-resident: its GB/s
    are cache, not HBM, figures. Every decode is checked against its input."""
    import torch

    from lossless_weight_compression_b200 import build_lib, synth, wcodec

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    build_lib.build()
    wc = wcodec.lib()
    stream = torch.cuda.current_stream(dev)
    peak, peak_kind = hbm_peak()
    l2_bytes = torch.cuda.get_device_properties(dev).L2_cache_size
    rows, ok_all = [], True

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        barrier(dist, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        barrier(dist, dev)
        return max_over_ranks(e0.elapsed_time(e1) / 1e3 / reps, dist, dev)

    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        for cfg in (1, 2, 3, 5):
            wl = synth.WORKLOADS[cfg]
            tensors = [t.view(-1).view(torch.int16) for _, t in wl.make(dev)]
            n = sum(t.numel() for t in tensors)
            counts = torch.zeros(256, dtype=torch.int64, device=dev)
            for t in tensors:
                counts += torch.bincount(((t.to(torch.int32) >> 7) & 0xFF), minlength=256)
            p = counts.double() / counts.sum()
            H = float(-(p[p > 0] * torch.log2(p[p > 0])).sum())
            for B in wl.blocks:
                for escape in (False, True):
                    enc = wcodec.CompressBatch(tensors, block=B, escape=escape)
                    enc.run()
                    torch.cuda.synchronize(dev)
                    sizes = enc.sizes()
                    outs = [torch.empty_like(t) for t in tensors]
                    status = torch.zeros(1, dtype=torch.int32, device=dev)
                    batch = wcodec.make_batch([(enc.buffers[k], sizes[k], outs[k], t.numel(), B)
                                               for k, t in enumerate(tensors)])
                    dec = wcodec.decompress_escape_batch if escape else wcodec.decompress_batch
                    reps = max(args.steps, int(2e9 // (2 * n)))  # a few hundred ms per case at most
                    t_enc = timed(enc.run, reps)
                    t_dec = timed(lambda: dec(batch, status), reps)
                    torch.cuda.synchronize(dev)
                    ok = (status.item() == 0 and enc.status.item() == 0
                          and all(torch.equal(a, b) for a, b in zip(tensors, outs)))
                    ok_all &= ok
                    C = sum(sizes)
                    moved = 2 * n + C
                    rows.append({
                        "workload": cfg, "name": wl.name, "block": B,
                        "stream": "escape-coded" if escape else "plain", "elements": n,
                        "ratio": 2 * n / C, "exponent_entropy_bits": H,
                        "entropy_bound_ratio": 16.0 / (8.0 + H),
                        "encode_ms": 1e3 * t_enc, "decode_ms": 1e3 * t_dec,
                        "encode_gbs_bf16_in": world * 2 * n / t_enc / 1e9,
                        "decode_gbs_bf16_out": world * 2 * n / t_dec / 1e9,
                        "decode_frac_of_peak": moved / t_dec / 1e9 / peak,
                        "encode_frac_of_peak": moved / t_enc / 1e9 / peak,
                        "l2_resident": moved + 2 * n <= l2_bytes,
                        "verified_bit_exact": ok})
                    del enc, outs, batch
            del tensors
    line = {
        "metric": "encode / decode GB/s and compression ratio per workload and block size",
        "value": None, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "u16", "data": "synthetic",
        "config": {"workload": "sweep: workloads 1, 2, 3, 5 at each of their block sizes, plain "
                               "and escape-coded streams", "peak_gbs": peak, "peak_kind": peak_kind,
                   "l2_bytes": l2_bytes},
        "sweep": rows, "clocks": clocks.summary(), "verified_bit_exact": ok_all,
        "gpu_launches": None,
    }
    if dist is not None:
        barrier(dist, dev)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok_all else 1


# ---------------------------------------------------------------------------
# next row: fused decode + matrix-vector products over the stack's linear weights
# ---------------------------------------------------------------------------
def run_dtype(args):
    """FP32 or FP16 weights: encode and decode of the first K decoder layers of the
    8B-shaped stack drawn in that dtype (same seeds as the BF16 stack). FP32
    tensors go through wc_compress_fp32 / wc_decompress_fp32, one launch each;
    FP16 tensors through the 16-bit batch path, one launch per direction."""
    import torch

    from lossless_weight_compression_b200 import build_lib, synth, wcodec

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    build_lib.build()
    wc = wcodec.lib()
    stream = torch.cuda.current_stream(dev)
    fp32 = args.workload == "fp32"
    dtype = torch.float32 if fp32 else torch.float16
    layers = args.gemv_layers or 4
    mats = [t for l in range(layers) for _, t in synth.layer_tensors(l, dev, rank_seed_base(rank), dtype)]
    n_all = sum(t.numel() for t in mats)
    esize = 4 if fp32 else 2
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    outs = [torch.empty_like(t) for t in mats]
    if fp32:
        comp = [wcodec.compress_fp32(t, BLOCK) for t in mats]
        torch.cuda.synchronize(dev)
        sizes = [c.size() for c in comp]
        wss = [wcodec.workspace_for(t.numel(), BLOCK, dev) for t in mats]

        def encode_all():
            for t, c, ws in zip(mats, comp, wss):
                rc = wc.wc_compress_fp32(t.data_ptr(), t.numel(), BLOCK, c.buffer.data_ptr(),
                                         c.buffer.numel(), c.nbytes.data_ptr(), ws.data_ptr(),
                                         ws.numel(), status.data_ptr(), stream.cuda_stream)
                if rc != 0:
                    raise RuntimeError("wc_compress_fp32: %s" % wc.wc_status_string(rc))

        def decode_all():
            for c, size, o in zip(comp, sizes, outs):
                rc = wc.wc_decompress_fp32(c.buffer.data_ptr(), size, o.data_ptr(), o.numel(),
                                           BLOCK, status.data_ptr(), stream.cuda_stream)
                if rc != 0:
                    raise RuntimeError("wc_decompress_fp32: %s" % wc.wc_status_string(rc))
        launches = 2 * len(mats)
        enc_kernel, dec_kernel = "encode_kernel<1,true>", "decode_kernel<1,true>"
    else:
        enc = wcodec.CompressBatch([t.view(-1).view(torch.int16) for t in mats], block=BLOCK)
        enc.run()
        torch.cuda.synchronize(dev)
        sizes = enc.sizes()
        batch = wcodec.make_batch([(enc.buffers[k], sizes[k], outs[k].view(-1).view(torch.int16),
                                    mats[k].numel(), BLOCK) for k in range(len(mats))])

        def encode_all():
            enc.run()

        def decode_all():
            wcodec.decompress_batch(batch, status)
        launches = 2
        enc_kernel, dec_kernel = "encode_kernel<512,false>", "decode_kernel<512,false>"

    def timed(fn):
        for _ in range(args.warmup):
            fn()
        barrier(dist, dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            fn()
        e1.record(stream)
        barrier(dist, dev)
        return max_over_ranks(e0.elapsed_time(e1) / 1e3 / args.steps, dist, dev)

    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        t_enc = timed(encode_all)
        t_dec = timed(decode_all)
    torch.cuda.synchronize(dev)
    ok = status.item() == 0 and all(torch.equal(a.view(-1), b.view(-1)) for a, b in zip(mats, outs))
    stream_bytes = sum(sizes)
    raw_bytes = esize * n_all
    peak, peak_kind = hbm_peak()
    moved = stream_bytes + raw_bytes
    name = "FP32" if fp32 else "FP16"
    line = {
        "metric": "decode GB/s (%s out) & %% HBM roofline; compression ratio" % name,
        "value": world * raw_bytes / t_dec / 1e9, "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * t_dec, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u32" if fp32 else "u16", "data": "synthetic",
        "config": {"workload": "first %d decoder layers of the 8B-shaped stack drawn in %s "
                               "(%d tensors, %d elements), block %d"
                               % (layers, name, len(mats), n_all, BLOCK),
                   "l2": "inputs larger than L2; no flush"},
        "roofline": {"bound": "hbm", "achieved": moved / t_dec / 1e9, "peak": peak, "unit": "GB/s",
                     "frac": moved / t_dec / 1e9 / peak, "peak_kind": peak_kind,
                     "kernel": dec_kernel, "algorithmic_bytes_per_launch": moved / (launches // 2),
                     "traffic": None},
        "compression": {"ratio": raw_bytes / stream_bytes, "stream_bytes": stream_bytes},
        "encode": {"ms_per_step": 1e3 * t_enc, "gbs_moved": moved / t_enc / 1e9,
                   "frac_of_peak": moved / t_enc / 1e9 / peak, "kernel": enc_kernel},
        "gpu_launches": args.steps * launches // 2,
        "clocks": clocks.summary(),
        "verified_bit_exact": ok,
    }
    if dist is not None:
        barrier(dist, dev)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


def run_gemv(args):
    """Fused decode + products over the 225 linear weight matrices of the
    8B-shaped stack (32 layers x 7 + LM head; the embedding is a lookup, not a
    product): wc_gemv_batch with n_vec activation vectors (gemv workload), or
    wc_gemm_batch on the tensor cores with `tokens` activation rows (gemm
    workload, one launch per 64 matrices); against torch's BF16 matmul (cuBLAS)
    on the same matrices, replayed from a CUDA graph."""
    import torch

    from lossless_weight_compression_b200 import build_lib, synth, wcodec

    world, rank, local = dist_env()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist = init_dist(world, "nccl")
    build_lib.build()
    wc = wcodec.lib()
    stream = torch.cuda.current_stream(dev)
    gemm = args.workload == "gemm"
    nv = args.tokens if gemm else args.n_vec
    if args.gemv_layers is None:
        mats = [(name, t) for name, t in synth.stack_tensors(dev, rank_seed_base(rank))
                if name != "embed_tokens"]
    else:  # a smaller case for profiling: the first layers only
        mats = [m for l in range(args.gemv_layers)
                for m in synth.layer_tensors(l, dev, rank_seed_base(rank))]
    weights = sum(t.numel() for _, t in mats)
    enc = wcodec.CompressBatch([t for _, t in mats], block=BLOCK, escape=args.escape_streams)
    enc.run()
    torch.cuda.synchronize(dev)
    sizes = enc.sizes()
    with ClockSampler(dev.index if dev.index is not None else 0) as clocks:
        res, ok = fused_phase(args, wc, wcodec, [t for _, t in mats], enc.buffers, sizes, nv, gemm,
                              stream, dist, dev, world, escape=args.escape_streams)
    what = "gemm" if gemm else "gemv"
    line = {
        "metric": "fused decode+%s weights/s (effective BF16 GB/s)" % what.upper(),
        "value": res["value"], "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": res["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "u16 weights, f32 accumulate", "data": "synthetic",
        "config": {"workload": "%s over %d linear weight matrices of the 8B-shaped stack "
                               "(%d weights), %s=%d, block %d, %s streams"
                               % (what, len(mats), weights, "tokens" if gemm else "n_vec", nv,
                                  BLOCK, res["stream"]),
                   "l2": "weights larger than L2; no flush"},
        "roofline": res["roofline"],
        "cublas_bf16": res["cublas_bf16"],
        "tflops": res["tflops"],
        "gpu_launches": res["gpu_launches"],
        "clocks": clocks.summary(),
        "verified_within_fp32_bound": ok,
    }
    if dist is not None:
        barrier(dist, dev)
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0 if ok else 1


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("wcodec", "reference"), default="wcodec")
    ap.add_argument("--workload", choices=("stack", "layer", "gemv", "gemm", "fp32", "fp16",
                                           "escape", "escape-layer", "sweep"),
                    default="stack",
                    help="stack: the 8B-shaped stack (the benchmark); layer: one decoder layer "
                         "(a smaller case for profiling); escape / escape-layer: the same as "
                         "escape-coded streams; sweep: workloads 1, 2, 3, 5 at each of their "
                         "block sizes, both stream kinds; gemv: fused decode + matrix-vector "
                         "products over the stack's linear weights; gemm: the same on the "
                         "tensor cores with --tokens activation rows; fp32 / fp16: encode and "
                         "decode of the first --gemv-layers (default 4) layers in that dtype")
    ap.add_argument("--tokens", type=int, default=64,
                    help="activation rows per product, 1..128 (gemm workload)")
    ap.add_argument("--n-vec", type=int, default=1, choices=(1, 2, 4),
                    help="activation vectors per product (gemv workload)")
    ap.add_argument("--gemv-layers", type=int, default=None,
                    help="gemv/gemm workload on the first K decoder layers only (a smaller case); "
                         "fp32/fp16 workloads: the number of layers (default 4)")
    ap.add_argument("--no-cpu-baseline", action="store_true",
                    help="skip timing the CPU oracle (for profiling runs)")
    ap.add_argument("--no-e2e", action="store_true",
                    help="skip the end-to-end (pinned host memory) measurement")
    ap.add_argument("--no-escape", action="store_true",
                    help="stack/layer workloads: skip the escape-coded streams' measurement")
    ap.add_argument("--no-tans", action="store_true",
                    help="stack/layer workloads: skip the tANS-coded streams' measurement")
    ap.add_argument("--fused-tokens", type=lambda v: [int(t) for t in v.split(",") if t],
                    default=[1, 16, 128],
                    help="stack/layer workloads: token counts of the fused decode+GEMM "
                         "measurement on the same streams (comma list; empty to skip)")
    ap.add_argument("--escape-streams", action="store_true",
                    help="gemm workload: multiply from escape-coded streams")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        log("note: fewer than 3 warm-up steps")
    if args.impl == "reference":
        return run_reference(args)
    if args.workload in ("gemv", "gemm"):
        return run_gemv(args)
    if args.workload in ("fp32", "fp16"):
        return run_dtype(args)
    if args.workload in ("escape", "escape-layer"):
        return run_escape(args)
    if args.workload == "sweep":
        return run_sweep(args)
    return run_wcodec(args)


if __name__ == "__main__":
    sys.exit(main())
