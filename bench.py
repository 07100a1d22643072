#!/usr/bin/env python3
"""Decode throughput of liblwc on B200.

Default workload (the largest single-GPU configuration): a Llama-3-70B-shaped
model (80 decoder layers of q 8192x8192, k/v 1024x8192, o 8192x8192, gate/up
28672x8192, down 8192x28672, plus the 128256x8192 embedding and LM head:
70,552,387,584 BF16 weights, N(0, sigma) with sigma ~ U(0.005, 0.03) per matrix
and 0.1 % outliers x20; synthetic, seeded, generated and compressed on the GPU)
held compressed with the DFloat11 codec in HBM (~94 GB). One step = one pass
over the model: every unit (embedding, 80 layers, LM head) decoded in order,
one layer-batched launch each, into two reusable BF16 buffers (ping-pong).
Metric: decoded BF16 GB/s (2 bytes per weight / step time), with the HBM
roofline fraction of the decode kernel and bits/weight.

Extra keys (one GPU): the Llama-3-8B layer (decode, codebook codec, device
encoders, FP32/FP16 element types, the decode-fused linear layer) and the
whole Llama-3-8B model with both codecs.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lwc|reference]
                    [--workload model70b|layer|layer70b|model8b|stress]

N > 1 (under torchrun): every rank decodes its own replica on its own GPU; no
data crosses GPUs (weak scaling); the reported time is the maximum over ranks.
--impl reference times the CPU oracle on the host cores instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import concurrent.futures as cf
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

import synth  # noqa: E402

METRIC = "decoded BF16 GB/s and % of HBM roofline (1\u00d7B200); bits/weight vs BF16"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0             # B200 HBM3e, nominal
PROFILE_TRAFFIC = os.path.join(ROOT, "profiles", "dram_traffic.txt")
DECODE_KERNEL = "df11_counted_kernel"   # blobs with stored chunk counts, the encoder's default
KERNEL_SOURCES = ("decode_dfloat11_b200/csrc/lwc_df11.cu", "decode_dfloat11_b200/csrc/lwc_df11_dev.cuh",
                  "decode_dfloat11_b200/csrc/lwc_device.cuh")


def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("lwc", "reference"), default="lwc")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-encode", action="store_true", help="skip the device-encoder timing")
    ap.add_argument("--no-elements", action="store_true", help="skip the FP32/FP16 DFloat11 decodes")
    ap.add_argument("--no-codebook", action="store_true")
    ap.add_argument("--no-linear", action="store_true", help="skip the decode-fused linear layer timing")
    ap.add_argument("--layer", type=int, default=None, help="layer seed (default: rank)")
    ap.add_argument("--workload", choices=("model70b", "layer", "layer70b", "model8b", "stress"),
                    default="model70b",
                    help="model70b (default) / model8b: the whole model resident compressed, decoded "
                         "layer by layer into ping-pong buffers; layer: one Llama-3-8B layer; layer70b: "
                         "one Llama-3-70B layer; stress: 256M-weight codebook and uniform-exponent tensors")
    ap.add_argument("--no-extras", action="store_true",
                    help="default workload only: skip the Llama-3-8B layer and model keys")
    ap.add_argument("--codec", choices=("dfloat11", "codebook"), default="dfloat11",
                    help="codec of the model workloads")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    if a.steps < 1:
        ap.error("--steps must be >= 1")
    return a


def kernel_sha() -> str:
    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def measured_tensor_peak():
    """Dense BF16 tensor-core peak (TFLOP/s): the burst cuBLAS figure of
    MEASURED_PEAKS.json (a kernel timed alone), else the fallback."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_BF16_TFLOPS, "fallback"


def mixed_roofline(bytes_moved: float, flops: float, ms: float, hbm_peak: float, tc_peak: float):
    """Roofline of a kernel that both streams bytes and runs the tensor cores:
    the bound is whichever of bytes / HBM peak and flops / tensor peak takes
    longer; both fractions are reported."""
    t_hbm = bytes_moved / (hbm_peak * 1e9)
    t_tc = flops / (tc_peak * 1e12)
    gbs = bytes_moved / (ms * 1e-3) / 1e9
    tfs = flops / (ms * 1e-3) / 1e12
    if t_hbm >= t_tc:
        head = {"bound": "hbm", "achieved": round(gbs, 1), "peak": hbm_peak, "unit": "GB/s",
                "frac": round(gbs / hbm_peak, 4)}
    else:
        head = {"bound": "tensor", "achieved": round(tfs, 1), "peak": tc_peak, "unit": "TFLOP/s",
                "frac": round(tfs / tc_peak, 4)}
    head.update({"hbm_frac": round(gbs / hbm_peak, 4), "tensor_frac": round(tfs / tc_peak, 4),
                 "algorithmic_bytes_per_call": int(bytes_moved), "flops_per_call": int(flops),
                 "target_ms": round(max(t_hbm, t_tc) * 1e3, 5)})
    return head


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def profiled_traffic(workload: str, alg_bytes_per_launch: float | None = None):
    """DRAM bytes (read + write) per launch of the decode kernel from the
    committed ncu summary, if it was taken on the current kernel source and
    this workload; else None. Lines: <kernel> <workload> <source sha> <bytes>
    [<algorithmic bytes of the captured launch>]. With the last field and
    alg_bytes_per_launch, the captured traffic is scaled to this run's average
    launch (traffic grows with the bytes a launch decodes)."""
    try:
        with open(PROFILE_TRAFFIC) as f:
            for line in f:
                parts = line.split()
                if len(parts) in (4, 5) and parts[0] == DECODE_KERNEL and parts[1] == workload \
                        and parts[2] == kernel_sha():
                    if len(parts) == 5 and alg_bytes_per_launch:
                        return int(round(int(parts[3]) * alg_bytes_per_launch / int(parts[4])))
                    return int(parts[3])
    except OSError:
        pass
    return None


def roofline_entry(alg_bytes_per_launch: float, launch_ms: float, traffic, peak_kind_pair, kernel=DECODE_KERNEL):
    """The roofline object: achieved = algorithmic bytes per launch / launch
    time, against the measured copy bandwidth (and, for context, nominal 8 TB/s)."""
    peak, peak_kind = peak_kind_pair
    achieved = alg_bytes_per_launch / (launch_ms * 1e-3) / 1e9
    return {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak, "unit": "GB/s",
            "frac": round(achieved / peak, 4), "traffic": traffic,
            "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs, a copy's bandwidth)"
            if peak_kind == "measured" else peak_kind,
            "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
            "algorithmic_bytes_per_launch": int(round(alg_bytes_per_launch)), "kernel": kernel,
            "launch_ms": round(launch_ms, 5)}


# ---------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={gpu_id}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if not self.proc:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except Exception:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, mx, reasons, power = [], [], set(), []
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for line in out.splitlines():
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


def gpu_id_for(device) -> str:
    import torch
    props = torch.cuda.get_device_properties(device)
    uuid = getattr(props, "uuid", None)
    if uuid is not None:
        s = str(uuid)
        return s if s.startswith("GPU-") else "GPU-" + s
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        return vis.split(",")[device.index or 0]
    return str(device.index or 0)


# ---------------------------------------------------------------- ranks

def rank_layer(rank: int, layer_arg) -> int:
    """Layer (seed) a rank decodes: its own, so replicas hold different data."""
    return layer_arg if layer_arg is not None else rank


def max_over_ranks(x: float, dist, device=None) -> float:
    """Largest value of x over all ranks (x itself without a process group)."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_gbs(world: int, bytes_per_rank: int, ms_per_step: float) -> float:
    """Aggregate GB/s when every rank moves bytes_per_rank per step and the
    step takes ms_per_step on the slowest rank."""
    return world * bytes_per_rank / (ms_per_step * 1e-3) / 1e9


# ---------------------------------------------------------------- setup

def make_layer(layer: int):
    names, tensors = [], []
    for name, t in synth.llama_layer_tensors(layer):
        names.append(name)
        tensors.append(synth.as_u16(t))
    return names, tensors


def encode_all(tensors, codec: str):
    from decode_dfloat11_b200 import lwc
    fn = lwc.lwc_encode_dfloat11 if codec == "df11" else lwc.lwc_encode_codebook
    with cf.ThreadPoolExecutor(max_workers=min(8, len(tensors))) as ex:
        return list(ex.map(fn, tensors))


def time_steps(step, steps: int, stream):
    import torch
    start = torch.cuda.Event(enable_timing=True)
    end = torch.cuda.Event(enable_timing=True)
    start.record(stream)
    for _ in range(steps):
        step()
    end.record(stream)
    end.synchronize()
    return start.elapsed_time(end)


def cpu_baseline(blobs, n_total: int, what: str = "the Llama-3-8B layer"):
    """The oracle decoder as it stands, single thread, on this host."""
    from oracle import df11 as odf
    t0 = time.perf_counter()
    n = 0
    for b in blobs:
        h = odf.B.unpack_header(b)
        odf.decode(b)
        n += h["n"]
        if time.perf_counter() - t0 > 30:
            break
    dt = time.perf_counter() - t0
    return {"value": round(2 * n / dt / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "sample": f"oracle bit-serial DFloat11 decode of {n:,} of the {n_total:,} weights of {what} "
                      f"(library-encoded blobs), one host thread, {dt:.2f} s"}


def _oracle_decode_worker(job) -> int:
    """Decode one piece of a blob that sits in a shared-memory segment:
    (segment name, offset, size, first block, end block); a block range of
    (0, 0) means the whole blob."""
    from multiprocessing import shared_memory

    from oracle import df11 as odf
    name, off, size, b0, b1 = job
    shm = shared_memory.SharedMemory(name=name)
    try:
        blob = np.ndarray((size,), dtype=np.uint8, buffer=shm.buf, offset=off)
        n = (odf.decode(blob) if (b0, b1) == (0, 0) else odf.decode_blocks(blob, b0, b1)).size
        del blob
    finally:
        shm.close()
    return int(n)


class OraclePool:
    """Spawned worker processes (no fork after the GPU was used), one per host
    core, that decode blobs with the oracle; the blobs sit in one
    shared-memory segment and each task is a range of a blob's blocks (about
    four tasks per worker), which the stored block offsets and gaps let any
    process decode on its own. ``decode_all()`` decodes every blob once and
    returns the weight count; waits are bounded."""

    def __init__(self, blobs):
        self.blobs = blobs
        try:   # the cores this process may run on (a container's CPU set), at most 32 workers
            cores = len(os.sched_getaffinity(0))
        except AttributeError:
            cores = os.cpu_count() or 1
        self.workers = max(1, min(cores, 32))

    def __enter__(self):
        import multiprocessing as mp
        from multiprocessing import shared_memory

        from oracle import blob as OB
        total = sum(b.size for b in self.blobs)
        self.shm = shared_memory.SharedMemory(create=True, size=max(1, total))
        weights = [int(OB.unpack_header(b)["n"]) for b in self.blobs]
        piece = max(1, sum(weights) // (4 * self.workers))   # about 4 pieces per worker
        jobs, off = [], 0
        for b, n in zip(self.blobs, weights):
            np.ndarray((b.size,), dtype=np.uint8, buffer=self.shm.buf, offset=off)[:] = b
            nb = int(OB.unpack_header(b).get("n_blocks", 0) or 0)
            if nb == 0:
                jobs.append((n, (self.shm.name, off, b.size, 0, 0)))
            else:   # block ranges of about `piece` weights, decoded independently
                k = max(1, min(nb, -(-n // piece)))
                cuts = [nb * i // k for i in range(k + 1)]
                jobs += [(n * (y - x) // nb, (self.shm.name, off, b.size, x, y)) for x, y in zip(cuts, cuts[1:])]
            off += b.size
        self.jobs = [j for _, j in sorted(jobs, key=lambda t: -t[0])]   # largest first
        self.pool = mp.get_context("spawn").Pool(self.workers)
        self._map([self.jobs[-1]] * self.workers)          # start the workers, import the oracle
        return self

    def _map(self, jobs) -> int:
        return sum(self.pool.map_async(_oracle_decode_worker, jobs, chunksize=1).get(timeout=600))

    def decode_all(self) -> int:
        return self._map(self.jobs)

    def __exit__(self, *exc):
        self.pool.terminate()
        self.pool.join()
        self.shm.close()
        self.shm.unlink()
        return False


def cpu_baseline_all_cores(blobs, n_total: int):
    """The same oracle decoder, one tensor per worker process, on the host's
    cores; timed with the workers already started."""
    import multiprocessing as mp
    try:
        with OraclePool(blobs) as pool:
            t0 = time.perf_counter()
            n = pool.decode_all()
            dt = time.perf_counter() - t0
            workers = pool.workers
    except mp.TimeoutError:
        return {"unavailable": "oracle worker processes did not finish within 600 s"}
    return {"value": round(2 * n / dt / 1e9, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
            "sample": f"oracle bit-serial DFloat11 decode of the whole layer ({n:,} weights) in block ranges "
                      f"on {workers} spawned workers (blobs in shared memory), {dt:.2f} s"}


# ---------------------------------------------------------------- our arm

def run_lwc(args, rank, world, local_rank, dist):
    import torch
    from decode_dfloat11_b200 import build as lwc_build
    from decode_dfloat11_b200 import lwc

    lwc_build.build()
    lwc.load()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    layer = rank_layer(rank, args.layer)

    names, tensors = make_layer(layer)
    n_total = sum(w.size for w in tensors)
    t_host = time.perf_counter()
    enc = encode_all(tensors, "df11")
    host_encode_s = time.perf_counter() - t_host
    descs = [d for d, _ in enc]
    blobs_h = [b for _, b in enc]
    blob_bytes = sum(b.size for b in blobs_h)
    blobs_d = [torch.from_numpy(b).to(device) for b in blobs_h]
    out = torch.empty(n_total, dtype=torch.bfloat16, device=device)   # the reusable layer buffer
    views, off = [], 0
    for w in tensors:
        views.append(out[off:off + w.size])
        off += w.size
    batch = lwc.Batch(descs, blobs_d, views)
    status = torch.zeros(1, dtype=torch.int32, device=device)
    groups = {(d.chunk_bytes, d.threads_per_block) for d in descs if not d.flags & 1}
    launches_per_step = len(groups) + sum(1 for d in descs if d.flags & 1 and d.n)

    def step():
        lwc.lwc_decode_dfloat11_batched(batch, stream=stream)

    # correctness of the very buffers being timed
    lwc.lwc_decode_dfloat11_batched(batch, d_status=status, stream=stream)
    torch.cuda.synchronize(device)
    for w, v in zip(tensors, views):
        if not torch.equal(v.view(torch.int16), torch.from_numpy(w.view(np.int16)).to(device)):
            raise SystemExit("decoded layer differs from its input")
    if int(status.item()):
        raise SystemExit(f"decoder reported status {int(status.item())}")

    # bring the GPU to its loaded clock, then the W warm-up steps, then K timed steps
    sampler = ClockSampler(gpu_id_for(device))
    t_heat = time.perf_counter()
    while time.perf_counter() - t_heat < 1.0:
        for _ in range(20):
            step()
        torch.cuda.synchronize(device)
    for _ in range(args.warmup):
        step()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    ms = time_steps(step, args.steps, stream)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms_per_step = max_over_ranks(ms, dist, device) / args.steps
    value = whole_job_gbs(world, 2 * n_total, ms_per_step)

    # roofline of the decode kernel (one launch per step here)
    peak, peak_kind = measured_peak()
    launch_ms = ms / (args.steps * launches_per_step)
    alg_bytes = (blob_bytes + 2 * n_total) / launches_per_step
    workload = "llama3-8b-layer-df11"
    roofline = roofline_entry(alg_bytes, launch_ms, profiled_traffic(workload, alg_bytes), (peak, peak_kind))

    result = {
        "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
        "data": "synthetic (seeded N(0, sigma) BF16, sigma ~ U(0.01, 0.04), 0.1% outliers x20)",
        "config": {"workload": workload, "tensors": names, "weights_per_gpu": n_total,
                   "compressed_bytes_per_gpu": blob_bytes,
                   "bits_per_weight": round(8 * blob_bytes / n_total, 4),
                   "size_vs_bf16": round(blob_bytes / (2 * n_total), 4),
                   "parallelism": f"replicas x{world} (each GPU decodes its own layer; no collective)",
                   "l2": f"no flush: {(blob_bytes + 2 * n_total) / 1e6:.0f} MB moved per step > 126 MB L2",
                   "chunk_bytes": descs[0].chunk_bytes, "threads_per_block": descs[0].threads_per_block},
        "roofline": roofline,
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks,
    }

    # codebook codec: the same layer in one batched launch, and a 256M-weight
    # stress tensor (U = 8192 Zipf(1.1) table, k = 13) as secondary figures
    if not args.no_codebook:
        cenc = encode_all(tensors, "codebook")
        cblobs = [torch.from_numpy(b).to(device) for _, b in cenc]
        cbatch = lwc.Batch([d for d, _ in cenc], cblobs, views)

        def cstep():
            lwc.lwc_decode_codebook_batched(cbatch, stream=stream)
        cstep()
        torch.cuda.synchronize(device)
        for w, v in zip(tensors, views):
            if not torch.equal(v.view(torch.int16), torch.from_numpy(w.view(np.int16)).to(device)):
                raise SystemExit("codebook-decoded layer differs from its input")
        for _ in range(args.warmup):
            cstep()
        cms = time_steps(cstep, args.steps, stream) / args.steps
        cbytes = sum(b.numel() for b in cblobs)
        result["codebook"] = {
            "workload": "llama3-8b-layer-codebook (one batched launch)",
            "value": round(2 * n_total / (cms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(cms, 5),
            "bits_per_weight": round(8 * cbytes / n_total, 4), "index_bits": [d.k for d, _ in cenc],
            "hbm_frac": round((cbytes + 2 * n_total) / (cms * 1e-3) / 1e9 / peak, 4)}
        del cblobs, cbatch
        ns = 1 << 28
        xs = synth.codebook_stress(8192, ns, seed=40 + 8192, device=device)
        sd, sb = lwc.lwc_encode_codebook(synth.as_u16(xs))
        sbd = torch.from_numpy(sb).to(device)
        sout = torch.empty(ns, dtype=torch.int16, device=device)
        lwc.lwc_decode_codebook(sd, sbd, sout, stream)
        torch.cuda.synchronize(device)
        if not torch.equal(sout, xs.view(torch.int16)):
            raise SystemExit("codebook stress decode differs from its input")
        del xs
        for _ in range(args.warmup):
            lwc.lwc_decode_codebook(sd, sbd, sout, stream)
        sms = time_steps(lambda: lwc.lwc_decode_codebook(sd, sbd, sout, stream), args.steps, stream) / args.steps
        result["codebook_stress"] = {
            "workload": f"codebook 256M weights, U={sd.U}, k={sd.k}, Zipf(1.1)",
            "value": round(2 * ns / (sms * 1e-3) / 1e9, 2), "unit": "GB/s", "ms_per_step": round(sms, 5),
            "bits_per_weight": round(sd.bits_per_weight, 4),
            "hbm_frac": round((sb.size + 2 * ns) / (sms * 1e-3) / 1e9 / peak, 4)}
        del sbd, sout

    # decode fused into the linear layer (token generation: M activation rows):
    # the layer's seven y = x W^T with the weights decoded in registers, one
    # batched call per codec, against decode-then-matmul and the uncompressed
    # BF16 matmul (torch), for context
    if not args.no_linear:
        from decode_dfloat11_b200.layers import encode_on_device
        lin = {"workload": "llama3-8b-layer: 7 x (y = x W^T), batched call, weights decoded in registers",
               "kernels": {"dfloat11": "df11_counted_linear_kernel", "codebook": "cb_linear_kernel"},
               "route": "layers.fused_linear (route auto) takes the fused kernel, except DFloat11 with "
                        "M > DF11_FUSED_MAX_M, where it decodes then multiplies"}
        src = [torch.from_numpy(w.view(np.int16)).to(device).view(torch.bfloat16).view(r, c)
               for w, (_, r, c) in zip(tensors, synth.LLAMA3_8B_LAYER)]
        for codec in ("dfloat11", "codebook"):
            enc_l = [encode_on_device(t, codec) for t in src]
            ld = [d for d, _ in enc_l]
            lb = [b for _, b in enc_l]
            lbytes = sum(b.numel() for b in lb)
            fn = lwc.lwc_linear_dfloat11_batched if codec == "dfloat11" else lwc.lwc_linear_codebook_batched
            dec = lwc.lwc_decode_dfloat11_batched if codec == "dfloat11" else lwc.lwc_decode_codebook_batched
            dbatch = lwc.Batch(ld, lb, views)
            for M in (1, 2, 4):
                xs = [synth.activations_bf16(M, t.shape[1], seed=500 + j, device=device) for j, t in enumerate(src)]
                ys = [torch.empty((M, t.shape[0]), dtype=torch.float32, device=device) for t in src]
                lbatch = lwc.LinearBatch(ld, lb, [t.shape[1] for t in src], xs, ys, M)
                fn(lbatch, stream=stream)
                torch.cuda.synchronize(device)
                for t, x, y in zip(src, xs, ys):   # consistency with torch on the same weights
                    ref = x.float() @ t.float().T
                    if not torch.allclose(y, ref, rtol=1e-3, atol=1e-3 * float(ref.abs().max())):
                        raise SystemExit(f"fused {codec} linear layer disagrees with torch")
                for _ in range(args.warmup):
                    fn(lbatch, stream=stream)
                fms = time_steps(lambda: fn(lbatch, stream=stream), args.steps, stream) / args.steps

                def unfused():
                    dec(dbatch, stream=stream)
                    for x, v, t in zip(xs, views, src):
                        torch.matmul(x, v.view(t.shape).T)
                for _ in range(args.warmup):
                    unfused()
                ums = time_steps(unfused, args.steps, stream) / args.steps
                dense = lambda: [torch.matmul(x, t.T) for x, t in zip(xs, src)]
                for _ in range(args.warmup):
                    dense()
                bms = time_steps(dense, args.steps, stream) / args.steps
                io = sum(2 * x.numel() + 4 * y.numel() for x, y in zip(xs, ys))
                ach = (lbytes + io) / (fms * 1e-3) / 1e9
                from decode_dfloat11_b200.layers import DF11_FUSED_MAX_M
                route = "decode" if codec == "dfloat11" and M > DF11_FUSED_MAX_M else "fused"
                lin[f"{codec}_M{M}"] = {
                    "fused_ms": round(fms, 5), "decode_then_matmul_ms": round(ums, 5),
                    "bf16_matmul_ms": round(bms, 5), "speedup_vs_decode_then_matmul": round(ums / fms, 3),
                    "layers_fused_linear_route": route,
                    "routed_speedup_vs_decode_then_matmul": round(ums / (fms if route == "fused" else ums), 3),
                    "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peak, "unit": "GB/s",
                                 "frac": round(ach / peak, 4), "algorithmic_bytes_per_call": lbytes + io}}
                del xs, ys, lbatch
            del enc_l, ld, lb, dbatch

        # the tensor-core product (prefill-size M): the weights in tile order,
        # each 128 x 64 tile decoded straight into the MMA's shared-memory
        # operand; against decode-then-matmul (row-major blobs) and the BF16 matmul
        from decode_dfloat11_b200.layers import TiledWeights
        tc_peak, _ = measured_tensor_peak()
        tw = TiledWeights(device)
        tidx = [tw.add(t) for t in src]
        tbytes = tw.compressed_bytes
        enc_d = [encode_on_device(t, "dfloat11") for t in src]
        dbatch = lwc.Batch([d for d, _ in enc_d], [b for _, b in enc_d], views)
        lin["kernels"]["dfloat11_tensor_core"] = "df11_gemm_kernel (tcgen05.mma, TMEM accumulator, x by TMA)"
        for M in (16, 64, 128, 256):
            xs = [synth.activations_bf16(M, t.shape[1], seed=700 + j, device=device) for j, t in enumerate(src)]
            ys = [torch.empty((M, t.shape[0]), dtype=torch.float32, device=device) for t in src]
            tb = lwc.LinearBatch(tw.descs, tw.blobs, [t.shape[1] for t in src], xs, ys, M)
            lwc.lwc_gemm_dfloat11_batched(tb, stream=stream)
            torch.cuda.synchronize(device)
            for t, x, y in zip(src, xs, ys):   # consistency with torch on the same weights
                ref = x.float() @ t.float().T
                if not torch.allclose(y, ref, rtol=1e-3, atol=1e-3 * float(ref.abs().max())):
                    raise SystemExit("tensor-core product disagrees with torch")
            for _ in range(args.warmup):
                lwc.lwc_gemm_dfloat11_batched(tb, stream=stream)
            gms = time_steps(lambda: lwc.lwc_gemm_dfloat11_batched(tb, stream=stream), args.steps, stream) / args.steps

            def unfused_tc():
                lwc.lwc_decode_dfloat11_batched(dbatch, stream=stream)
                for x, v, t in zip(xs, views, src):
                    torch.mm(x, v.view(t.shape).T, out_dtype=torch.float32)
            for _ in range(args.warmup):
                unfused_tc()
            ums = time_steps(unfused_tc, args.steps, stream) / args.steps
            dense = lambda: [torch.mm(x, t.T, out_dtype=torch.float32) for x, t in zip(xs, src)]
            for _ in range(args.warmup):
                dense()
            bms = time_steps(dense, args.steps, stream) / args.steps
            io = sum(2 * x.numel() + 4 * y.numel() for x, y in zip(xs, ys))
            lin[f"dfloat11_tc_M{M}"] = {
                "tc_ms": round(gms, 5), "decode_then_matmul_ms": round(ums, 5), "bf16_matmul_ms": round(bms, 5),
                "speedup_vs_decode_then_matmul": round(ums / gms, 3),
                "roofline": mixed_roofline(tbytes + io, 2.0 * M * n_total, gms, peak, tc_peak)}
            del xs, ys, tb
        del tw, enc_d, dbatch

        # the same for the codebook codec (the layer's matrices grouped by index width)
        twc = TiledWeights(device, codec="codebook")
        cidx = [twc.add(t) for t in src]
        cbytes = twc.compressed_bytes
        enc_c = [encode_on_device(t, "codebook") for t in src]
        cbatch = lwc.Batch([d for d, _ in enc_c], [b for _, b in enc_c], views)
        groups = {}
        for i in cidx:
            groups.setdefault(twc.descs[i].k, []).append(i)
        lin["kernels"]["codebook_tensor_core"] = "cb_gemm_kernel<k> (tcgen05.mma, TMEM accumulator, x by TMA)"
        for M in (16, 64, 128, 256):
            xs = [synth.activations_bf16(M, t.shape[1], seed=900 + j, device=device) for j, t in enumerate(src)]
            ys = [torch.empty((M, t.shape[0]), dtype=torch.float32, device=device) for t in src]
            cbs = [lwc.LinearBatch([twc.descs[i] for i in g], [twc.blobs[i] for i in g],
                                   [src[i].shape[1] for i in g], [xs[i] for i in g], [ys[i] for i in g], M)
                   for g in groups.values()]

            def cgemm():
                for b in cbs:
                    lwc.lwc_gemm_codebook_batched(b, stream=stream)
            cgemm()
            torch.cuda.synchronize(device)
            for t, x, y in zip(src, xs, ys):
                ref = x.float() @ t.float().T
                if not torch.allclose(y, ref, rtol=1e-3, atol=1e-3 * float(ref.abs().max())):
                    raise SystemExit("codebook tensor-core product disagrees with torch")
            for _ in range(args.warmup):
                cgemm()
            gms = time_steps(cgemm, args.steps, stream) / args.steps

            def unfused_cb():
                lwc.lwc_decode_codebook_batched(cbatch, stream=stream)
                for x, v, t in zip(xs, views, src):
                    torch.mm(x, v.view(t.shape).T, out_dtype=torch.float32)
            for _ in range(args.warmup):
                unfused_cb()
            ums = time_steps(unfused_cb, args.steps, stream) / args.steps
            io = sum(2 * x.numel() + 4 * y.numel() for x, y in zip(xs, ys))
            lin[f"codebook_tc_M{M}"] = {
                "tc_ms": round(gms, 5), "decode_then_matmul_ms": round(ums, 5),
                "speedup_vs_decode_then_matmul": round(ums / gms, 3), "launches": len(cbs),
                "roofline": mixed_roofline(cbytes + io, 2.0 * M * n_total, gms, peak, tc_peak)}
            del xs, ys, cbs
        del twc, enc_c, cbatch
        result["linear"] = lin
        del src

    # DFloat11 for the other float formats: a gate-shaped FP32 and FP16 matrix
    if not args.no_elements:
        rows, cols = 14336, 4096
        ne = rows * cols
        res_el = {}
        for label, elem in (("fp32", lwc.LWC_ELEM_FP32), ("fp16", lwc.LWC_ELEM_FP16)):
            if elem == lwc.LWC_ELEM_FP32:
                xe = synth.normal_bf16((rows, cols), seed=7000, sigma=0.02).float()
                xe = xe + torch.randn(xe.shape, generator=torch.Generator().manual_seed(7001)) * 1e-5
                xh = xe.numpy().view(np.uint32).reshape(-1)
                out_e = torch.empty(ne, dtype=torch.int32, device=device)
            else:
                xh = synth.as_u16(synth.normal_fp16((rows, cols), seed=7002, sigma=0.02, outlier_frac=1e-3))
                out_e = torch.empty(ne, dtype=torch.int16, device=device)
            de, be = lwc.lwc_encode_dfloat11_elements(xh, elem)
            bd = torch.from_numpy(be).to(device)
            lwc.lwc_decode_dfloat11(de, bd, out_e, stream)
            torch.cuda.synchronize(device)
            if not np.array_equal(out_e.cpu().numpy().view(xh.dtype), xh):
                raise SystemExit(f"{label} decode differs from its input")
            for _ in range(args.warmup):
                lwc.lwc_decode_dfloat11(de, bd, out_e, stream)
            ems_e = time_steps(lambda: lwc.lwc_decode_dfloat11(de, bd, out_e, stream), args.steps, stream) / args.steps
            esz = xh.dtype.itemsize
            res_el[label] = {
                "workload": f"{label} {rows}x{cols} matrix (Llama-3-8B gate shape), DFloat11 elements",
                "value": round(esz * ne / (ems_e * 1e-3) / 1e9, 2), "unit": "GB/s decoded",
                "ms_per_step": round(ems_e, 5), "bits_per_weight": round(8 * be.size / ne, 4),
                "size_vs_uncompressed": round(be.size / (esz * ne), 4),
                "hbm_frac": round((be.size + esz * ne) / (ems_e * 1e-3) / 1e9 / peak, 4)}
            del bd, out_e, xh
        result["elements"] = res_el

    # device encoders (load-time path): the same layer, already on the GPU,
    # compressed there; blobs must equal the host encoder's byte for byte
    if not args.no_encode:
        from decode_dfloat11_b200.layers import encode_on_device
        src = [torch.from_numpy(w.view(np.int16)).to(device) for w in tensors]
        work = torch.empty(lwc.lwc_encode_device_workspace_bytes(max(w.size for w in tensors)),
                           dtype=torch.uint8, device=device)
        enc_res = {"workload": "llama3-8b-layer, 7 tensors on the GPU, plan + write per tensor",
                   "host_df11_ms": round(host_encode_s * 1e3, 1), "host_threads": min(8, len(tensors))}
        for codec in ("dfloat11", "codebook"):
            got = [encode_on_device(t, codec, workspace=work) for t in src]
            ref = blobs_h if codec == "dfloat11" else [b for _, b in encode_all(tensors, "codebook")]
            if not all(np.array_equal(b.cpu().numpy(), r) for (_, b), r in zip(got, ref)):
                raise SystemExit(f"device {codec} encoder differs from the host encoder")
            del got
            reps = 3
            torch.cuda.synchronize(device)
            t0 = time.perf_counter()
            for _ in range(reps):
                for t in src:
                    encode_on_device(t, codec, workspace=work)
            torch.cuda.synchronize(device)
            ems_enc = (time.perf_counter() - t0) / reps * 1e3
            enc_res[f"{codec}_ms"] = round(ems_enc, 3)
            enc_res[f"{codec}_gbs"] = round(2 * n_total / (ems_enc * 1e-3) / 1e9, 1)
        enc_res["same_bytes_as_host"] = True
        result["encode"] = enc_res
        del src, work

    # end to end through the C ABI with host buffers: pinned blobs -> device,
    # decode, decoded layer -> pinned host, every step (layers.HostPipeline:
    # tensor i's upload, i-1's decode and i-2's read-back overlap on three
    # streams; the timing events sit on the decode stream, which waits for the
    # last read-back before the end event).
    if not args.no_e2e:
        from decode_dfloat11_b200.layers import HostPipeline
        pipe = HostPipeline(descs, [torch.from_numpy(b) for b in blobs_h], "dfloat11", device)

        def estep():
            pipe.run(stream)
        for _ in range(3):
            estep()
        e_steps = max(3, min(args.steps, 20))
        torch.cuda.synchronize(device)
        ems = time_steps(estep, e_steps, stream) / e_steps
        torch.cuda.synchronize(device)
        for w, off in zip(tensors, pipe.offsets):
            if not torch.equal(pipe.host_out.view(torch.int16)[off:off + w.size], torch.from_numpy(w.view(np.int16))):
                raise SystemExit("end-to-end output differs from its input")
        ev = whole_job_gbs(world, 2 * n_total, max_over_ranks(ems, dist, device))
        result["e2e"] = {"value": round(ev, 3), "unit": "GB/s", "h2d_bytes_per_step": pipe.h2d_bytes,
                         "d2h_bytes_per_step": pipe.d2h_bytes, "ms_per_step": round(ems, 4), "steps": e_steps,
                         "pipeline": "layers.HostPipeline: per-tensor H2D / decode / D2H on three streams"}
        del pipe

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(blobs_h, n_total)
        result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(blobs_h, n_total)
    return result


# ---------------------------------------------------------------- model workloads

def model_units(which: str, device):
    """(name, generator) per unit of a Llama-3-shaped model; generators make
    the unit's seeded tensors on the given device. layer70b: decoder layer 0
    of the Llama-3-70B model alone."""
    if which == "model8b":
        hidden, shapes, layers, sig, off = (synth.LLAMA3_8B_HIDDEN, synth.LLAMA3_8B_LAYER,
                                            synth.LLAMA3_8B_LAYERS, (0.01, 0.04), 0)
    else:
        hidden, shapes, layers, sig, off = (synth.LLAMA3_70B_HIDDEN, synth.LLAMA3_70B_LAYER,
                                            synth.LLAMA3_70B_LAYERS, (0.005, 0.03), synth.SEED_70B_OFFSET)
    layer_units = [(f"layer{L}", lambda L=L: [t for _, t in synth.llama_layer_tensors(
        L, shapes, sig, off, device=device)]) for L in range(layers)]
    if which == "layer70b":
        return layer_units[:1]
    return ([("embed", lambda: [synth.llama_embedding("embed", hidden, sig, off, device=device)])] + layer_units +
            [("lm_head", lambda: [synth.llama_embedding("lm_head", hidden, sig, off, device=device)])])


MODEL_WORKLOADS = {"model70b": "llama3-70b-model", "model8b": "llama3-8b-model", "layer70b": "llama3-70b-layer"}


def run_model(args, rank, world, local_rank, dist, which=None, codec=None, baselines=True):
    """Whole models (Llama-3-8B or Llama-3-70B shapes; or one 70B layer)
    resident compressed in HBM; one step decodes every unit in order (one
    batched launch each) into two reusable BF16 buffers. With `baselines`
    (the default line): the oracle timed on one layer's blobs on this host,
    and an end-to-end pass of one layer through layers.HostPipeline."""
    import torch
    from decode_dfloat11_b200 import build as lwc_build
    from decode_dfloat11_b200 import lwc
    from decode_dfloat11_b200.layers import ResidentModel

    which = which or args.workload
    codec = codec or args.codec
    lwc_build.build()
    lwc.load()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    units = model_units(which, device)
    model = ResidentModel(codec, device)
    t0 = time.perf_counter()
    work = None
    for name, gen in units:   # generated on the GPU and compressed there (device encoder)
        tensors = gen()
        need = max(lwc.lwc_encode_device_workspace_bytes(t.numel()) for t in tensors)
        if work is None or work.numel() < need:
            work = torch.empty(need, dtype=torch.uint8, device=device)
        model.add_layer_from_device(name, tensors, workspace=work)
        del tensors
    del work
    model.finalize()
    setup_s = time.perf_counter() - t0
    n_total, blob_bytes = model.weights, model.compressed_bytes
    status = torch.zeros(1, dtype=torch.int32, device=device)

    # every unit checked once against its regenerated tensors
    for i, (name, gen) in enumerate(units):
        model.decode(i, i % 2, stream, status)
        expect = gen()
        for v, t in zip(model.views(i, i % 2), expect):
            if not torch.equal(v.view(torch.int16), t.view(torch.int16)):
                raise SystemExit(f"decoded {name} differs from its input")
        del expect
    if int(status.item()):
        raise SystemExit(f"decoder reported status {int(status.item())}")

    def step():
        for i in range(len(units)):
            model.decode(i, i % 2, stream)

    sampler = ClockSampler(gpu_id_for(device))
    for _ in range(args.warmup):
        step()
    if dist:
        dist.barrier()
    torch.cuda.synchronize(device)
    ms = time_steps(step, args.steps, stream)
    torch.cuda.synchronize(device)
    if dist:
        dist.barrier()
    clocks = sampler.stop()
    ms_per_step = max_over_ranks(ms, dist, device) / args.steps
    peak_pair = measured_peak()
    launches = len(units)   # one batched launch per unit (every unit has several exponents)
    launch_ms = ms / (args.steps * launches)
    alg_per_launch = (blob_bytes + 2 * n_total) / launches
    wl = f"{MODEL_WORKLOADS[which]}-{codec}"
    traffic = profiled_traffic("llama3-70b-layer-dfloat11", alg_per_launch) \
        if which in ("model70b", "layer70b") and codec == "dfloat11" else None
    result = {
        "metric": METRIC,
        "value": round(whole_job_gbs(world, 2 * n_total, ms_per_step), 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "u16",
        "data": "synthetic (seeded N(0, sigma) BF16 + 0.1% outliers x20, generated on the GPU)",
        "config": {"workload": wl, "units": len(units),
                   "weights_per_gpu": n_total, "compressed_bytes_per_gpu": blob_bytes,
                   "bits_per_weight": round(8 * blob_bytes / n_total, 4),
                   "size_vs_bf16": round(blob_bytes / (2 * n_total), 4),
                   "buffers": "2 x largest unit (ping-pong)",
                   "setup_s": round(setup_s, 1), "setup": "tensors generated and compressed on the GPU",
                   "l2": f"no flush: {(blob_bytes + 2 * n_total) / 1e9:.1f} GB moved per step > 126 MB L2",
                   "parallelism": f"replicas x{world} (each GPU decodes its own copy; no collective)"},
        "roofline": roofline_entry(alg_per_launch, launch_ms, traffic, peak_pair,
                                   DECODE_KERNEL if codec == "dfloat11" else "cb_decode_kernel"),
        "gpu_launches": args.steps * launches,
        "clocks": clocks,
    }

    if baselines and codec == "dfloat11" and which != "model8b":
        li = next(i for i, (name, _) in enumerate(units) if name == "layer0")
        layer = model.layers[li]
        host_blobs = [b.cpu().numpy() for b in layer["blobs"]]
        n_layer = sum(layer["n"])
        if not args.no_e2e:
            # end to end through the C ABI with host buffers, one layer per step:
            # pinned blobs -> device, decode, decoded layer -> pinned host
            from decode_dfloat11_b200.layers import HostPipeline
            pipe = HostPipeline(layer["descs"], [torch.from_numpy(b) for b in host_blobs], "dfloat11", device)
            for _ in range(3):
                pipe.run(stream)
            e_steps = max(3, min(args.steps, 10))
            torch.cuda.synchronize(device)
            ems = time_steps(lambda: pipe.run(stream), e_steps, stream) / e_steps
            torch.cuda.synchronize(device)
            expect = units[li][1]()
            for t, off in zip(expect, pipe.offsets):
                if not torch.equal(pipe.host_out.view(torch.int16)[off:off + t.numel()], t.reshape(-1).view(torch.int16).cpu()):
                    raise SystemExit("end-to-end output differs from its input")
            del expect
            ev = whole_job_gbs(world, 2 * n_layer, max_over_ranks(ems, dist, device))
            result["e2e"] = {"value": round(ev, 3), "unit": "GB/s", "h2d_bytes_per_step": pipe.h2d_bytes,
                             "d2h_bytes_per_step": pipe.d2h_bytes, "ms_per_step": round(ems, 4), "steps": e_steps,
                             "sample": "one step = decoder layer 0 of the model (7 matrices, "
                                       f"{n_layer:,} weights) from pinned host blobs to pinned host BF16",
                             "pipeline": "layers.HostPipeline: per-tensor H2D / decode / D2H on three streams"}
            del pipe
        if rank == 0 and world == 1 and not args.no_cpu_baseline:
            result["cpu_baseline"] = cpu_baseline(host_blobs, n_layer, "one Llama-3-70B layer")
            result["cpu_baseline_all_cores"] = cpu_baseline_all_cores(host_blobs, n_layer)
    del model
    torch.cuda.empty_cache()
    return result


# ---------------------------------------------------------------- stress tensors

def run_stress(args, rank, world, local_rank, dist):
    """256M-weight stress tensors, each generated and compressed on
    the GPU and decoded K times: codebook tables of U = 256 / 4096 / 8192 /
    65536 entries with Zipf(1.1) frequencies (k = 8 / 12 / 13 / 16; also
    16384, 32768 and 40000 for k = 14, 15 and a k = 16 table that is not the
    identity: U = 65536 means every pattern, a table the decoder copies
    through), and the
    DFloat11 edge case of uniformly random patterns (all 256 exponents, 8-bit
    codes: an expansion)."""
    import torch
    from decode_dfloat11_b200 import build as lwc_build
    from decode_dfloat11_b200 import lwc
    from decode_dfloat11_b200.layers import encode_on_device

    lwc_build.build()
    lwc.load()
    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    stream = torch.cuda.current_stream(device)
    peak, peak_kind = measured_peak()
    n = 1 << 28
    cases = [("codebook", U) for U in (256, 4096, 8192, 16384, 32768, 40000, 65536)] + [("dfloat11", None)]
    rows, max_ms = {}, 0.0
    for codec, U in cases:
        x = synth.codebook_stress(U, n, seed=40 + U + rank, device=device) if U else \
            synth.uniform_patterns(n, seed=44 + rank, device=device)
        d, blob = encode_on_device(x, codec)
        out = torch.empty(n, dtype=torch.int16, device=device)
        dec = lwc.lwc_decode_codebook if codec == "codebook" else lwc.lwc_decode_dfloat11
        dec(d, blob, out, stream)
        torch.cuda.synchronize(device)
        if not torch.equal(out, x.view(torch.int16)):
            raise SystemExit(f"stress {codec} U={U} decode differs from its input")
        del x
        for _ in range(args.warmup):
            dec(d, blob, out, stream)
        ms = time_steps(lambda: dec(d, blob, out, stream), args.steps, stream) / args.steps
        ms = max_over_ranks(ms, dist, device)
        max_ms = max(max_ms, ms)
        key = f"codebook_U{U}" if U else "dfloat11_uniform_exponents"
        rows[key] = {"k": d.k if U else None, "bits_per_weight": round(d.bits_per_weight, 4),
                     "ms": round(ms, 5), "decoded_gbs": round(2 * n / (ms * 1e-3) / 1e9, 1),
                     "hbm_frac": round((d.total_bytes + 2 * n) / (ms * 1e-3) / 1e9 / peak, 4)}
        del blob, out
    first = rows["codebook_U8192"]
    return {
        "metric": "decoded BF16 GB/s (codebook U=8192 stress tensor; all config-4 cases in 'cases')",
        "value": round(world * first["decoded_gbs"], 2), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": first["ms"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u16",
        "data": "synthetic (Zipf(1.1) draws from U-entry tables; uniform 16-bit patterns)",
        "config": {"workload": "stress-256M", "weights_per_gpu": n, "parallelism": f"replicas x{world}",
                   "l2": "no flush: >= 805 MB moved per decode > 126 MB L2", "peak_source": peak_kind},
        "cases": rows, "gpu_launches": args.steps * len(cases),
    }


# ---------------------------------------------------------------- reference arm

def run_reference(args):
    """The CPU oracle as it stands, on this host's cores, for the same
    workload and metric as our arm, each step a bounded sample of it: for the
    whole-model workloads one matrix of layer 0 (the q matrix; generated on
    the CPU with the same recipe), for the Llama-3-8B layer the whole layer
    (its q matrix alone when more than 200 steps are asked for), decoded in
    block ranges on one spawned worker process per core."""
    from decode_dfloat11_b200 import build as lwc_build
    from decode_dfloat11_b200 import lwc
    lwc_build.build()
    if args.workload in ("model70b", "layer70b", "model8b"):
        seventy = args.workload != "model8b"
        shapes = synth.LLAMA3_70B_LAYER if seventy else synth.LLAMA3_8B_LAYER
        sig = (0.005, 0.03) if seventy else (0.01, 0.04)
        off = synth.SEED_70B_OFFSET if seventy else 0
        _, q = next(iter(synth.llama_layer_tensors(0, shapes, sig, off)))
        use = [synth.as_u16(q)]
        what = f"layer 0's q matrix ({use[0].size:,} weights, generated on the CPU with the same recipe)"
        workload = f"{MODEL_WORKLOADS[args.workload]}-dfloat11"
    else:
        _, tensors = make_layer(args.layer or 0)
        whole = args.steps + args.warmup <= 200
        use = tensors if whole else tensors[:1]
        what = "the whole Llama-3-8B layer" if whole else "the Llama-3-8B layer's q matrix"
        workload = "llama3-8b-layer-df11"
    blobs = [lwc.lwc_encode_dfloat11(t)[1] for t in use]
    n = sum(t.size for t in use)
    with OraclePool(blobs) as pool:
        for _ in range(args.warmup):
            pool.decode_all()
        t0 = time.perf_counter()
        for _ in range(args.steps):
            pool.decode_all()
        dt = (time.perf_counter() - t0) / args.steps
        workers = pool.workers
    value = 2 * n / dt / 1e9
    sample = (f"oracle bit-serial DFloat11 decode of {what} per step, in block ranges on "
              f"{workers} spawned workers")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "u16", "data": "synthetic",
        "config": {"workload": workload, "sample": what},
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": workers, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0
    dist = None
    if world > 1:
        import datetime
        import torch
        import torch.distributed as tdist
        torch.cuda.set_device(local_rank)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                 device_id=torch.device("cuda", local_rank))
        dist = tdist
    try:
        if args.workload == "layer":
            result = run_lwc(args, rank, world, local_rank, dist)
        elif args.workload == "stress":
            result = run_stress(args, rank, world, local_rank, dist)
        else:
            result = run_model(args, rank, world, local_rank, dist)
            if args.workload == "model70b" and world == 1 and not args.no_extras:
                # the other workloads' figures, on the same GPU, after the 70B model is freed
                import argparse as _ap
                sub = _ap.Namespace(**{**vars(args), "no_e2e": False, "no_cpu_baseline": True})
                layer = run_lwc(sub, rank, world, local_rank, dist)
                result["llama3_8b_layer"] = {k: v for k, v in layer.items()
                                             if k not in ("metric", "n_gpus", "steps", "warmup", "higher_is_better",
                                                          "scaling", "vs_baseline", "dtype", "data")}
                m8 = {}
                for codec in ("dfloat11", "codebook"):
                    r = run_model(sub, rank, world, local_rank, dist, which="model8b", codec=codec, baselines=False)
                    m8[codec] = {"value": r["value"], "unit": r["unit"], "ms_per_step": r["ms_per_step"],
                                 "bits_per_weight": r["config"]["bits_per_weight"],
                                 "weights": r["config"]["weights_per_gpu"], "roofline": r["roofline"],
                                 "clocks": r["clocks"]}
                result["llama3_8b_model"] = {"workload": "llama3-8b-model (32 layers + embedding + LM head), "
                                                         "decoded layer by layer into ping-pong buffers", **m8}
        if rank == 0:
            print(json.dumps(result), flush=True)
    finally:
        if dist:
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
