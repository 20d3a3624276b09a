#!/usr/bin/env python3
"""Benchmark of the MXFP8 attention forward hot path on B200.

One step is one pass of the whole path over one batch of synthetic input already resident
in HBM: varlen metadata, MXFP8 quantization of Q and K (and V in bf16 PV mode), the
unscaled E4M3 cast of V (fp8 PV mode), and the attention forward. `value` is attention
TFLOPS (sum of 4 * Sq * Sk * H * 128 over sequences, every rank) divided by the step time;
the `roofline` object reports the attention kernel alone against the measured dense FP8
peak, and `e2e` repeats the step with host buffers (pinned H2D of Q/K/V, D2H of O/LSE every
step, the copies of neighbouring steps overlapping this step's compute on two copy streams).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

For N > 1 run under torch.distributed.run: every rank processes its own copy of the
workload (weak scaling; sequences and heads are independent, so there is no collective on
the data path). `--impl reference` times the CPU oracle on a bounded sample instead.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

DEFAULT_WORKLOAD = "video_s32768_h24_fp8pv"
METRIC = "MXFP8 attn-fwd TFLOPS (4*Sq*Sk*H*d) & % of dense FP8 peak; quantize GB/s"
NOMINAL_FP8_TFLOPS = 4500.0          # dense, per GPU (context)
FP8_OVER_BF16 = 2.0                  # nominal dense FP8 / BF16 tensor ratio
FALLBACK_BF16_BURST = 1590.0         # used only when MEASURED_PEAKS.json is absent
FALLBACK_HBM_GBS = 6650.0

# DRAM traffic of one attention launch, from an ncu capture of the same command (the capture
# summarised beside this kernel's profile). Valid only for the kernel source whose hash is
# recorded; any change to the kernel makes it null until re-captured.
TRAFFIC = {
    # workload: (sha256 of the kernel's sources [:16], dram bytes read + written per launch)
    "video_s32768_h24_fp8pv": ("388ff0548a182d31", 310078464 + 174111744),
    "dense_4x2048_h16": ("85f4f6c42fb74a08", 68298752 + 3575808),
    "cross_varlen_outliers_h32": ("85f4f6c42fb74a08", 3567325696 + 47040768),
}

# The source files of the attention kernel each PV mode runs, and that kernel's name.
KERNEL_SOURCES = {
    "fp8": (["attn_fwd_pp.cuh", "attn_fwd.cuh", "ptx.cuh"], "attn_fwd_pp_kernel"),
    "mxfp8": (["attn_fwd_pp.cuh", "attn_fwd.cuh", "ptx.cuh"], "attn_fwd_pp_kernel"),
    "bf16": (["attn_fwd_pp.cuh", "attn_fwd.cuh", "ptx.cuh", "dequantize.cuh"],
             "attn_fwd_pp_kernel (+ dequantize_mxfp8_kernel for V, timed with it)"),
    "bf16v": (["attn_fwd_pp.cuh", "attn_fwd.cuh", "ptx.cuh"], "attn_fwd_pp_kernel"),
}


def kernel_hash(pv_mode: str) -> str:
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[pv_mode][0]:
        with open(os.path.join(ROOT, "precision_attention_forward_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:16]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except (OSError, ValueError):
        return {"hbm_gbs": FALLBACK_HBM_GBS, "bf16_tflops": FALLBACK_BF16_BURST}, "fallback"


def attention_flops(lq, lk, heads) -> float:
    """4 * Sq * Sk * H * 128 summed over the (query, key) sequence pairs; a single query sequence
    with several key sequences is the shared-query workload (the query set pairs with each)."""
    if len(lq) == 1 and len(lk) > 1:
        return float(sum(4.0 * lq[0] * b * heads * 128 for b in lk))
    return float(sum(4.0 * a * b * heads * 128 for a, b in zip(lq, lk)))


def quantizer_bytes(tokens, heads, in_bytes, scale_blocks) -> float:
    return float(tokens) * heads * 128 * (in_bytes + 1) + float(scale_blocks) * heads * 512


def smi_index_of(local_rank: int) -> int:
    """nvidia-smi / NVML index of this rank's GPU (CUDA_VISIBLE_DEVICES maps CUDA ordinals)."""
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = vis.split(",")
        if local_rank < len(ids) and ids[local_rank].strip().isdigit():
            return int(ids[local_rank])
    return local_rank


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons of one GPU during the timed region.

    NVML is polled every ~2 ms from a background thread, and only samples between mark("start")
    and mark("end") (host times around the synchronised timed region) count, so even a timed
    region of a few hundred milliseconds yields tens of samples. Without NVML it falls back to
    `nvidia-smi -lms 100` over the whole run.
    """

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    # NVML clock-event reason bits reported by name (the rest are idle / application settings).
    REASON_BITS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
                   0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown"}

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []
        self.t = None
        self.nvml = None
        self.samples = []
        self.marks = {}
        self.halt = False

    def mark(self, which: str):
        self.marks[which] = time.perf_counter()

    def start(self):
        try:
            import pynvml
            pynvml.nvmlInit()
            self.h = pynvml.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nvml = pynvml
        except Exception:
            self.nvml = None
        if self.nvml is not None:
            self.t = threading.Thread(target=self._poll, daemon=True)
            self.t.start()
            return
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.QUERY}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.t = threading.Thread(target=self._read, daemon=True)
        self.t.start()

    def _poll(self):
        nv = self.nvml
        while not self.halt:
            try:
                sm = nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                self.samples.append((time.perf_counter(), float(sm), int(rs)))
            except Exception:
                pass
            time.sleep(0.002)

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.nvml is not None:
            self.halt = True
            if self.t:
                self.t.join(timeout=2)
            try:
                self.nvml.nvmlShutdown()
            except Exception:
                pass
            t0, t1 = self.marks.get("start"), self.marks.get("end")
            sel = [x for x in self.samples if (t0 is None or x[0] >= t0) and (t1 is None or x[0] <= t1)]
            inside = bool(sel)
            if not sel:
                sel = self.samples
            reasons = set()
            for _, _, rs in sel:
                for bit, name in self.REASON_BITS.items():
                    if rs & bit:
                        reasons.add(name)
            return {"sm_mhz": statistics.median(x[1] for x in sel) if sel else None,
                    "sm_max_mhz": float(self.max_mhz), "reasons": sorted(reasons), "samples": len(sel),
                    "source": "NVML, ~2 ms polling" + (" inside the timed region" if inside else " over the run")}
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx.append(float(parts[2]))
            except ValueError:
                continue
            for n, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm), "source": "nvidia-smi -lms 100 over the run"}


def cpu_oracle_sample(w, seconds: float, seed: int = 0):
    """Time the CPU oracle on a bounded sample of the workload: for one head at a time,
    quantize that head's K and V (or cast V), quantize a block of query rows, and run the
    fp64 attention of those rows over all keys. Returns (tflops, desc, cores, elapsed)."""
    from oracle import attention as oatt
    from oracle import mxfp8 as omx

    lq, lk = wl.lengths(w)
    q = wl.make_tensor(w, "q")
    k = wl.make_tensor(w, "k")
    v = wl.make_tensor(w, "v")
    cu_q = np.concatenate([[0], np.cumsum(lq)])
    cu_k = np.concatenate([[0], np.cumsum(lk)])
    rows_per = 128
    done_flops = 0.0
    units = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        i = units % len(lk)
        iq = 0 if w.shared_q else i   # a shared query set pairs with every K/V sequence
        h = (units // len(lq)) % w.heads
        k0, k1 = cu_k[i], cu_k[i + 1]
        kp, ke = omx.quantize_rows(k[k0:k1, h].astype(np.float64), w.scaling_mode)
        kh = (omx.e4m3_decode(kp).reshape(-1, 4, 32) * np.ldexp(1.0, ke)[..., None]).reshape(-1, 128)
        if w.pv_mode == "fp8":
            vh = omx.e4m3_decode(omx.cast_e4m3(v[k0:k1, h]))
        elif w.pv_mode == "bf16v":
            vh = v[k0:k1, h].astype(np.float64)
        elif w.pv_mode == "mxfp8":
            vpt, vst = omx.quantize_mxfp8_varlen_tokens(v[k0:k1, h][:, None, :], [k1 - k0], w.scaling_mode)
            vh = omx.dequantize_mxfp8_tokens(vpt, vst, [k1 - k0], 1)[:, 0]
        else:
            vp, ve = omx.quantize_rows(v[k0:k1, h].astype(np.float64), w.scaling_mode)
            vh = (omx.e4m3_decode(vp).reshape(-1, 4, 32) * np.ldexp(1.0, ve)[..., None]).reshape(-1, 128)
        r0 = cu_q[iq] + (units * rows_per) % max(1, lq[iq] - rows_per + 1)
        r1 = min(cu_q[iq + 1], r0 + rows_per)
        qp, qe = omx.quantize_rows(q[r0:r1, h].astype(np.float64), w.scaling_mode)
        qh = (omx.e4m3_decode(qp).reshape(-1, 4, 32) * np.ldexp(1.0, qe)[..., None]).reshape(-1, 128)
        oatt.attend_block(qh, kh, vh, p_mode={"fp8": "fp8", "mxfp8": "mxfp8"}.get(w.pv_mode, "exact"))
        done_flops += 4.0 * (r1 - r0) * (k1 - k0) * 128
        units += 1
    elapsed = time.perf_counter() - t0
    try:
        from threadpoolctl import threadpool_info
        cores = max([d.get("num_threads", 1) for d in threadpool_info()] + [1])
    except Exception:  # pragma: no cover
        cores = os.cpu_count() or 1
    desc = (f"{units} units of {rows_per} query rows x all keys of one (sequence, head), each with that "
            f"head's K/V quantization, fp64 numpy oracle")
    return done_flops / elapsed / 1e12, desc, cores, elapsed


def cpu_quantizer_sample(w, x, lens, payload_dev, scales_dev, in_bytes: int, seconds: float):
    """Time the CPU oracle's MXFP8 quantizer on a bounded sample of one input tensor: 4096-token
    chunks (128-aligned, so each is a sequence of its own with the same scale atoms) of the packed
    sequences in order, until `seconds` have passed. Algorithmic bytes as for the GPU quantizer
    (in_bytes + 1 per element, 512 per (128-token block, head) atom). Every byte of the chunks it
    quantized is compared with the GPU's payload and scales of the same tensor from this run.
    Returns (MB/s, description, bit_exact, elapsed)."""
    from oracle import meta as ometa
    from oracle import mxfp8 as omx

    m = ometa.from_lengths(lens)
    H = x.shape[1]
    chunks = []
    for i in range(m.num_seqs):
        n, c0 = int(m.lengths[i]), int(m.cu_seqlens[i])
        for t0 in range(0, n, 4096):
            chunks.append((i, c0 + t0, min(n, t0 + 4096) - t0, int(m.scale_off[i]) + t0 // 128))
    done, exact, nbytes = 0, True, 0.0
    t0 = time.perf_counter()
    results = []
    while done < len(chunks) and (done == 0 or time.perf_counter() - t0 < seconds):
        _, row0, rows, _ = chunks[done]
        results.append(omx.quantize_mxfp8_varlen(x[row0:row0 + rows], [rows], w.scaling_mode))
        nbytes += rows * H * 128 * (in_bytes + 1) + ((rows + 127) // 128) * H * 512
        done += 1
    elapsed = time.perf_counter() - t0
    for (_, row0, rows, b0), (ref_p, ref_s) in zip(chunks[:done], results):
        got_p = payload_dev[row0:row0 + rows].cpu().numpy()
        got_s = scales_dev[b0 * H * 512:b0 * H * 512 + ref_s.size].cpu().numpy()
        exact = exact and np.array_equal(got_p, ref_p) and np.array_equal(got_s, ref_s)
    desc = (f"{done} chunks of up to 4096 tokens x {H} heads of Q ({'fp32' if in_bytes == 4 else 'bf16'}), "
            f"fp64 numpy oracle quantizer ({w.scaling_mode}), each compared byte for byte with the GPU's")
    return nbytes / elapsed / 1e6, desc, exact, elapsed


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    lq, lk = wl.lengths(w)
    per_step = max(1.0, float(os.environ.get("LPFA_REF_STEP_SECONDS", "3.0")))
    for _ in range(args.warmup):
        cpu_oracle_sample(w, per_step)
    vals, times, descs, cores = [], [], None, 1
    for _ in range(args.steps):
        tf, desc, cores, el = cpu_oracle_sample(w, per_step)
        vals.append(tf)
        times.append(el)
        descs = desc
    value = statistics.median(vals)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000.0 * statistics.mean(times),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": config_dict(w, lq, lk, args.gpus),
        "cpu_baseline": {"value": value, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": descs},
        "e2e": {"value": value, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Ranks:
    """Host-side bookkeeping across the ranks of a run (one process per GPU): a barrier and a
    max over ranks of a float. There is no collective on the data path; the runs are replicas.

    ``device`` is where the reduction tensor lives: the rank's GPU under NCCL, the CPU under
    gloo (the CPU tests).
    """

    def __init__(self, world: int, device, sync_cuda: bool = True):
        self.world = world
        self.device = device
        self.sync_cuda = sync_cuda

    def barrier(self):
        import torch
        import torch.distributed as dist

        if self.world > 1:
            dist.barrier()
        if self.sync_cuda:
            torch.cuda.synchronize()

    def max(self, x: float) -> float:
        if self.world == 1:
            return float(x)
        import torch
        import torch.distributed as dist

        t = torch.tensor([x], dtype=torch.float64, device=self.device)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())


def job_tflops(flops_per_rank: float, world: int, ms_per_step: float) -> float:
    """Whole-job throughput: every rank processes flops_per_rank per step (weak scaling), and
    the step time is the slowest rank's."""
    return flops_per_rank * world / (ms_per_step * 1e-3) / 1e12


def l2_exceeded(lk, heads) -> bool:
    """K alone (bf16) exceeds the 126 MB L2, so no step finds its inputs in L2."""
    return float(np.sum(lk)) * heads * 128 * 2 > 126e6


def config_dict(w, lq, lk, n):
    return {
        "workload": w.name, "description": w.description, "num_seqs": int(w.num_seqs),
        "seq_len_q": int(max(lq)), "seq_len_k": int(max(lk)), "total_tokens_q": int(np.sum(lq)),
        "total_tokens_k": int(np.sum(lk)), "heads": w.heads, "head_dim": 128, "pv_mode": w.pv_mode,
        "in_dtype": w.in_dtype, "scaling_mode": w.scaling_mode, "global_batch": int(w.num_seqs) * n,
        "shared_q": bool(w.shared_q),
        "parallelism": f"replicas{n}" if n > 1 else "single",
        "l2": "inputs larger than L2 (no flush)" if l2_exceeded(lk, w.heads)
              else "L2 flushed between steps (256 MB write), step time from per-step events",
    }


def run_backward(args, w):
    """--pass bwd: the attention backward (lpfa_attn_bwd_varlen) on the workload, one GPU.

    A step is one backward call (its three kernels) on inputs already in HBM: MXFP8 Q/K/V in the
    head_dim orientation, the forward's O and LSE, a seeded BF16 dO. value = algorithmic
    TFLOPS, 10 * Sq * Sk * H * 128 (the five products; the dQ kernel recomputes S and dP, which
    is not counted); the products run as BF16 MMAs, so the peak is the measured BF16 burst.
    """
    import torch

    import precision_attention_forward_b200 as lp

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    stream = torch.cuda.current_stream()
    lq, lk = wl.lengths(w)
    H = w.heads
    flops = 2.5 * attention_flops(lq, lk, H)
    peaks, peak_src = load_peaks()
    host = {x: wl.make_tensor(w, x) for x in "qkv"}
    mq = lp.lpfa_varlen_meta_from_lengths(lq, device=dev)
    mk = lp.lpfa_varlen_meta_from_lengths(lk, device=dev)
    q8, qs = lp.lpfa_quantize_mxfp8_varlen(wl.to_torch(host["q"], wl.tensor_dtype(w, "q"), device=dev), mq, w.scaling_mode)
    k8, ks = lp.lpfa_quantize_mxfp8_varlen(wl.to_torch(host["k"], wl.tensor_dtype(w, "k"), device=dev), mk, w.scaling_mode)
    v8, vs = lp.lpfa_quantize_mxfp8_varlen(wl.to_torch(host["v"], "bf16" if w.pv_mode == "fp8" else w.in_dtype, device=dev),
                                           mk, w.scaling_mode)
    out, lse = lp.lpfa_attn_fwd_varlen(q8, qs, k8, ks, v8, vs, mq, mk, pv_mode="bf16")
    g = np.random.default_rng(7)
    dout = wl.to_torch(wl.round_to_bf16(g.standard_normal(out.shape, dtype=np.float32)), "bf16", device=dev)
    flush = not l2_exceeded(lk, H)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None
    sampler = ClockSampler(smi_index_of(0))
    sampler.start()
    for _ in range(args.warmup):
        lp.lpfa_attn_bwd_varlen(q8, qs, k8, ks, v8, vs, out, dout, lse, mq, mk)
    torch.cuda.synchronize()
    sampler.mark("start")
    times = []
    for _ in range(args.steps):
        if flush:
            flush_buf.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        lp.lpfa_attn_bwd_varlen(q8, qs, k8, ks, v8, vs, out, dout, lse, mq, mk)
        b.record(stream)
        times.append((a, b))
    torch.cuda.synchronize()
    sampler.mark("end")
    clocks = sampler.stop()
    st, detail = lp.lpfa_device_status()
    if st != lp.LPFA_OK:
        raise RuntimeError(f"kernel reported status {st} (site {detail})")
    ms = sum(a.elapsed_time(b) for a, b in times) / args.steps
    value = flops / (ms * 1e-3) / 1e12
    bf16_peak = peaks.get("bf16_tflops", FALLBACK_BF16_BURST)
    cfg = config_dict(w, lq, lk, 1)
    cfg["pass"] = "backward (dQ BF16, dK/dV BF16; MXFP8 Q/K/V head_dim orientation)"
    print(json.dumps({
        "metric": "MXFP8 attn-bwd TFLOPS (10*Sq*Sk*H*d)", "value": value, "unit": "TFLOPS", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": cfg,
        "roofline": {"bound": "tensor", "achieved": value, "peak": bf16_peak, "unit": "TFLOP/s",
                     "frac": value / bf16_peak, "traffic": None,
                     "peak_source": f"{peak_src} bf16 burst", "kernel": "attn_bwd_d_kernel + attn_bwd_dkdv_kernel + attn_bwd_dq_kernel",
                     "flops_per_launch": flops},
        "e2e": None, "gpu_launches": 3 * args.steps, "clocks": clocks, "cpu_baseline": None,
    }))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=sorted(wl.WORKLOADS))
    ap.add_argument("--impl", default="lpfa", choices=["lpfa", "reference"])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--pass", dest="which", default="fwd", choices=["fwd", "bwd"],
                    help="bwd: time the attention backward on one GPU instead of the forward step")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "lpfa":
        sys.stderr.write("note: fewer than 3 warm-up steps; numbers are for smoke use only\n")
    w = wl.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)
    if args.which == "bwd":
        return run_backward(args, w)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local_rank))

    import precision_attention_forward_b200 as lp

    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.current_stream()
    lq, lk = wl.lengths(w)
    H = w.heads
    flops = attention_flops(lq, lk, H)

    # Inputs, resident in HBM.
    host = {x: wl.make_tensor(w, x) for x in "qkv"}
    dts = {x: wl.tensor_dtype(w, x) for x in "qkv"}
    dev_in = {x: wl.to_torch(host[x], dts[x], device=dev) for x in "qkv"}
    Tq, Tk = int(np.sum(lq)), int(np.sum(lk))
    To = Tq * len(lk) if w.shared_q else Tq   # output rows
    mq0 = lp.lpfa_varlen_meta_from_lengths(lq, device=dev)
    sbq, sbk = mq0.total_scale_blocks, lp.lpfa_varlen_meta_from_lengths(lk, device=dev).total_scale_blocks
    qp = torch.empty((Tq, H, 128), dtype=torch.uint8, device=dev)
    kp = torch.empty((Tk, H, 128), dtype=torch.uint8, device=dev)
    vp = torch.empty((Tk, H, 128), dtype=torch.uint8, device=dev) if w.pv_mode != "bf16v" else None
    qs = torch.empty(sbq * H * 512, dtype=torch.uint8, device=dev)
    ks = torch.empty(sbk * H * 512, dtype=torch.uint8, device=dev)
    vs = torch.empty(sbk * H * 512, dtype=torch.uint8, device=dev) if w.pv_mode in ("bf16", "mxfp8") else None
    out = torch.empty((To, H, 128), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((H, To), dtype=torch.float32, device=dev)
    # bf16 PV: the workspace where V is dequantized to BF16 once per step.
    ws_bytes = lp.lpfa_attn_fwd_workspace_bytes(lp.lpfa_varlen_meta_fill_host(lk), H, w.pv_mode)
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev) if ws_bytes else False

    def step(ins, timing=None, result=None):
        o_dst, l_dst = result if result is not None else (out, lse)
        mq = lp.lpfa_varlen_meta_from_lengths(lq, device=dev)
        mk = lp.lpfa_varlen_meta_from_lengths(lk, device=dev)
        if timing is not None:
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
        lp.lpfa_quantize_mxfp8_varlen(ins["q"], mq, w.scaling_mode, payload=qp, scales=qs)
        lp.lpfa_quantize_mxfp8_varlen(ins["k"], mk, w.scaling_mode, payload=kp, scales=ks)
        if w.pv_mode == "fp8":
            lp.lpfa_cast_e4m3(ins["v"], out=vp)
        elif w.pv_mode == "bf16":
            lp.lpfa_quantize_mxfp8_varlen(ins["v"], mk, w.scaling_mode, payload=vp, scales=vs)
        elif w.pv_mode == "mxfp8":   # V in the token orientation
            lp.lpfa_quantize_mxfp8_varlen(ins["v"], mk, w.scaling_mode, payload=vp, scales=vs, orientation="tokens")
        if timing is not None:
            c = torch.cuda.Event(enable_timing=True)
            c.record(stream)
        v_in = ins["v"] if w.pv_mode == "bf16v" else vp   # BF16 V goes to the kernel as is
        attn = lp.lpfa_attn_fwd_shared_q if w.shared_q else lp.lpfa_attn_fwd_varlen
        attn(qp, qs, kp, ks, v_in, vs, mq, mk, pv_mode=w.pv_mode, out=o_dst, lse=l_dst, workspace=ws)
        if timing is not None:
            b.record(stream)
            timing.append((a, c, b))
        return {"bf16v": 3, "bf16": 5}.get(w.pv_mode, 4)  # kernels launched

    ranks = Ranks(world, dev)
    barrier = ranks.barrier
    max_over_ranks = ranks.max

    sampler = ClockSampler(smi_index_of(local_rank))
    sampler.start()
    # Workloads whose inputs fit in L2 get it flushed before every step (a 256 MB write outside
    # the step's own events); the step time is then the sum of the per-step event intervals.
    flush = not l2_exceeded(lk, w.heads)
    flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if flush else None

    def timed_step(timing=None):
        if flush:
            flush_buf.zero_()
        return step(dev_in, timing)

    for _ in range(args.warmup):
        timed_step()
    barrier()
    sampler.mark("start")
    timing = []
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches = 0
    start.record(stream)
    for _ in range(args.steps):
        launches += timed_step(timing)
    end.record(stream)
    barrier()
    sampler.mark("end")
    clocks = sampler.stop()
    total_ms = max_over_ranks(sum(a.elapsed_time(b) for a, c, b in timing) if flush else start.elapsed_time(end))
    quant_ms = sum(a.elapsed_time(c) for a, c, b in timing) / args.steps
    attn_ms = sum(c.elapsed_time(b) for a, c, b in timing) / args.steps
    attn_ms = max_over_ranks(attn_ms)
    quant_ms = max_over_ranks(quant_ms)
    st, detail = lp.lpfa_device_status()
    if st != lp.LPFA_OK:
        raise RuntimeError(f"kernel reported status {st} (site {detail})")

    ms_per_step = total_ms / args.steps
    value = job_tflops(flops, world, ms_per_step)

    # End to end through the public API with host buffers. Each step copies its Q/K/V in from
    # pinned host memory and its O/LSE out, pipelined the way a serving loop would run it: the
    # next step's inputs are copied in (copy stream) and the previous step's results copied out
    # (a second copy stream) while this step computes, into double-buffered device tensors. The
    # timed region spans the first step's input copy to the last step's output copy.
    e2e = None
    if not args.no_e2e:
        pinned = {x: dev_in[x].cpu().pin_memory() for x in "qkv"}
        o_host = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
        l_host = [torch.empty(lse.shape, dtype=lse.dtype).pin_memory() for _ in range(2)]
        ins_dev = [{x: torch.empty_like(dev_in[x]) for x in "qkv"} for _ in range(2)]
        res_dev = [(torch.empty_like(out), torch.empty_like(lse)) for _ in range(2)]
        h2d_s, d2h_s = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
        h2d = sum(t.numel() * t.element_size() for t in pinned.values()) + 2 * 4 * (len(lq) + 1) * 2
        d2h = o_host[0].numel() * o_host[0].element_size() + l_host[0].numel() * l_host[0].element_size()

        def run_e2e(n, start_ev=None):
            h2d_done, comp_done, d2h_done = [None] * n, [None] * n, [None] * n

            def copy_in(i):
                if start_ev is not None:
                    h2d_s.wait_event(start_ev)
                if i >= 2:
                    h2d_s.wait_event(comp_done[i - 2])   # step i - 2 has finished reading the buffer
                with torch.cuda.stream(h2d_s):
                    for x in "qkv":
                        ins_dev[i % 2][x].copy_(pinned[x], non_blocking=True)
                    ev = torch.cuda.Event()
                    ev.record(h2d_s)
                h2d_done[i] = ev

            copy_in(0)
            for i in range(n):
                if i + 1 < n:
                    copy_in(i + 1)
                stream.wait_event(h2d_done[i])
                if i >= 2:
                    stream.wait_event(d2h_done[i - 2])   # step i - 2's results have been copied out
                step(ins_dev[i % 2], result=res_dev[i % 2])
                ce = torch.cuda.Event()
                ce.record(stream)
                comp_done[i] = ce
                d2h_s.wait_event(ce)
                with torch.cuda.stream(d2h_s):
                    o_host[i % 2].copy_(res_dev[i % 2][0], non_blocking=True)
                    l_host[i % 2].copy_(res_dev[i % 2][1], non_blocking=True)
                    de = torch.cuda.Event()
                    de.record(d2h_s)
                d2h_done[i] = de
            stream.wait_event(d2h_done[n - 1])
            return (n - 1) % 2

        run_e2e(max(2, args.warmup // 2))
        barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        ne = max(3, args.steps // 2)
        e0.record(stream)
        last = run_e2e(ne, start_ev=e0)
        e1.record(stream)
        barrier()
        e_ms = max_over_ranks(e0.elapsed_time(e1)) / ne
        # The pipelined steps must give exactly the results of the resident-input step.
        step(dev_in)
        torch.cuda.synchronize()
        same = bool(torch.equal(o_host[last].view(torch.int16), out.cpu().view(torch.int16)) and
                    torch.equal(l_host[last].view(torch.int32), lse.cpu().view(torch.int32)))
        e2e = {"value": job_tflops(flops, world, e_ms), "unit": "TFLOPS", "ms_per_step": e_ms,
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "pipelined": True,
               "results_match_resident_step": same}

    peaks, peak_src = load_peaks()
    # The attention kernel runs at full SM clock (it is not power capped like a dense GEMM), so
    # the burst GEMM figure is the denominator: the larger, more conservative of the two.
    fp8_peak = peaks.get("bf16_tflops", FALLBACK_BF16_BURST) * FP8_OVER_BF16
    achieved = flops / (attn_ms * 1e-3) / 1e12
    tr = TRAFFIC.get(w.name)
    traffic = tr[1] if tr and tr[0] == kernel_hash(w.pv_mode) else None
    qbytes = quantizer_bytes(Tq, H, 2 if dts["q"] == "bf16" else 4, sbq) + \
        quantizer_bytes(Tk, H, 2 if dts["k"] == "bf16" else 4, sbk) + \
        (Tk * H * 128 * 3.0 if w.pv_mode == "fp8" else
         0.0 if w.pv_mode == "bf16v" else quantizer_bytes(Tk, H, 2 if dts["v"] == "bf16" else 4, sbk))

    if rank == 0:
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            tf, desc, cores, el = cpu_oracle_sample(w, float(os.environ.get("LPFA_CPU_SECONDS", "15")))
            qmbs, qdesc, qexact, qel = cpu_quantizer_sample(w, host["q"], lq, qp, qs,
                                                            2 if dts["q"] == "bf16" else 4,
                                                            float(os.environ.get("LPFA_CPU_QUANT_SECONDS", "5")))
            cpu = {"value": tf, "unit": "TFLOPS", "cores": cores, "kind": "oracle", "sample": desc,
                   "seconds": el,
                   "quantizer": {"value": qmbs, "unit": "MB/s", "sample": qdesc, "seconds": qel,
                                 "bit_exact_vs_gpu": bool(qexact)}}
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "e4m3", "data": "synthetic",
            "config": config_dict(w, lq, lk, world),
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": fp8_peak, "unit": "TFLOP/s",
                         "frac": achieved / fp8_peak, "traffic": traffic,
                         "peak_source": f"{peak_src} bf16 burst x {FP8_OVER_BF16:g} (nominal FP8/BF16 ratio)",
                         "kernel": KERNEL_SOURCES[w.pv_mode][1], "flops_per_launch": flops},
            "attn_kernel_ms": attn_ms,
            "attn_pct_nominal_fp8": 100.0 * achieved / NOMINAL_FP8_TFLOPS,
            "quantize": {"ms_per_step": quant_ms, "bytes_per_step": qbytes,
                         "gbs": qbytes / (quant_ms * 1e-3) / 1e9,
                         "frac_hbm": qbytes / (quant_ms * 1e-3) / 1e9 / peaks.get("hbm_gbs", FALLBACK_HBM_GBS)},
            "e2e": e2e,
            "gpu_launches": launches,
            "clocks": clocks,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
