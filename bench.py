"""Benchmark of the action-aware causal attention hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl native|reference]
                    [--workload 480p-long-session]

One step is one pass of the whole hot path over one batch: build the mask
metadata (per-token descriptors, tile schedule, unmasked-pair count) on the
host and upload it, run the attention forward of the current segment over the
cache, and append the segment's K/V to the cache (the cache is rolled back to
its prior segments afterwards so every step sees the same session length).

Metric: effective attention TFLOP/s counting unmasked work only,
4 * 128 * heads * A per call, A the unmasked query-key pairs per head (Eq. 6 of
the Hy-Nomas report). Rank 0 prints one JSON line. With N > 1 (torchrun) each
rank runs an independent replica of the workload (no data-path collective:
the path has no exchange step) and `value` is the sum over ranks divided by
the slowest rank's device time.
"""
from __future__ import annotations

import argparse
import dataclasses
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from segment_causal_masked_b200 import workloads as W  # noqa: E402

METRIC = "effective attention TFLOP/s (unmasked work) and % of B200 dense BF16 peak"
WORKLOADS = {
    "480p-long-session": W.session_480p_long,
    "480p-single-turn": W.session_480p_single_turn,
    "720p-step": W.session_720p,
    "packed-360k": W.packed_360k,
    "tiny-packed": W.tiny_packed,
    # inference options (sliding window of 4 earlier segments; a quarter of
    # the video blocks kept, drawn at random with a fixed seed per pair of
    # query tiles)
    "480p-long-session-window4": lambda: W.with_history(W.session_480p_long(), 4),
    "480p-long-session-blocks25": lambda: W.with_random_blocks(W.session_480p_long(), 0.25, 25,
                                                               group=2),
    # INT8 KV cache (codes + per-row scales, quantised by the append kernel)
    "480p-long-session-int8": lambda: dataclasses.replace(W.session_480p_long(),
                                                          name="480p-long-session-int8"),
}
WORKLOADS["480p-single-turn-int8"] = lambda: dataclasses.replace(W.session_480p_single_turn(),
                                                                 name="480p-single-turn-int8")
# the INT8 cache with a workspace that also holds a bf16 copy of it: the call
# dequantises once (an HBM-bound copy) and runs the bf16 kernel on the copy
WORKLOADS["480p-long-session-int8-copy"] = lambda: dataclasses.replace(
    W.session_480p_long(), name="480p-long-session-int8-copy")
INT8_WORKLOADS = {"480p-long-session-int8", "480p-single-turn-int8", "480p-long-session-int8-copy"}
INT8_COPY_WORKLOADS = {"480p-long-session-int8-copy"}
# the backward of the packed training batch (the forward that produces O and
# LSE runs once, untimed; a step is one backward call)
WORKLOADS["packed-360k-bwd"] = lambda: dataclasses.replace(W.packed_360k(), name="packed-360k-bwd")
WORKLOADS["packed-64k-bwd"] = lambda: dataclasses.replace(W.packed_360k(budget=64_000),
                                                          name="packed-64k-bwd")
BWD_WORKLOADS = {"packed-360k-bwd", "packed-64k-bwd"}
# one denoising step of a 480p segment as the distilled model runs it: the
# metadata built and uploaded once, four attention calls (one per NFE, each
# with that NFE's own current-segment Q, K and V, seed + nfe) against the same
# cache, then the append of the segment's K/V (the last NFE's)
WORKLOADS["480p-single-turn-4nfe"] = lambda: dataclasses.replace(
    W.session_480p_single_turn(), name="480p-single-turn-4nfe")
NFE_WORKLOADS = {"480p-single-turn-4nfe": 4}
# the camera cross-attention of one 480p segment (out = x + softmax(q k_camᵀ)
# v_cam): an HBM-bound call with its own metric, GB/s of algorithmic bytes
WORKLOADS["camera-xattn-480p"] = W.camera_480p
CAMERA_WORKLOADS = {"camera-xattn-480p"}
CAMERA_METRIC = "camera cross-attention HBM GB/s (algorithmic bytes) and % of measured copy bandwidth"
CAMERA_INPUT_SETS = 4   # (q, x, out) sets rotated over the steps: 4 x 149 MB > L2
# a timed call this long runs at the power-capped clock: its fraction is taken
# against the sustained bf16 peak, shorter calls against the burst peak
SUSTAINED_CALL_MS = 500.0
BWD_FLOP_FACTOR = 2.5   # five products per visible pair against the forward's two
KERNEL_SOURCES = {
    "attn_fwd_kernel": ["segment_causal_masked_b200/csrc/sca_kernels.cu",
                        "segment_causal_masked_b200/csrc/sca_ptx.cuh",
                        "segment_causal_masked_b200/csrc/sca_internal.h"],
    "camera_xattn_kernel": ["segment_causal_masked_b200/csrc/sca_camera.cu",
                            "segment_causal_masked_b200/csrc/sca_camera.h",
                            "segment_causal_masked_b200/csrc/sca_ptx.cuh"],
}


def kernel_hash(kernel: str = "attn_fwd_kernel") -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def effective_flops(problem, unmasked_pairs: int) -> float:
    return 4.0 * W.HEAD_DIM * problem.heads * unmasked_pairs


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return dict(json.load(f), source="measured")
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
            "source": "fallback"}


def stored_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f)
    e = d.get(kernel, {}).get(workload)
    if not e or e.get("kernel_hash") != kernel_hash(kernel):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.rows = []
        self.proc = None
        self.thread = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-i", str(self.gpu), "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append([x.strip() for x in line.split(",")])

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        if self.thread:
            self.thread.join(timeout=2)
        return clock_summary(self.rows)


def clock_summary(rows) -> dict:
    """Median SM clock, the maximum clock and every throttle reason seen
    active, from nvidia-smi rows in ClockSampler.FIELDS order (rows that do
    not parse are skipped)."""
    sm, mx, reasons = [], [], set()
    names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
    for r in rows:
        try:
            sm.append(float(r[1]))
            mx.append(float(r[2]))
        except (ValueError, IndexError):
            continue
        for n, v in zip(names, r[5:9]):
            if v.strip().lower() == "active":
                reasons.add(n)
    return {"sm_mhz": statistics.median(sm) if sm else None,
            "sm_max_mhz": max(mx) if mx else None,
            "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# the CPU oracle (baseline and the reference arm only)
# ---------------------------------------------------------------------------

class OracleSample:
    """The oracle on `rows` query rows (spread evenly over the query tiles) and
    `heads` head(s) of the workload, inputs drawn once."""

    def __init__(self, problem, rows: int, heads: int = 1, seed: int = 7, int8: bool = False,
                 backward: bool = False):
        import numpy as np
        import torch

        from oracle import cache as ocache
        from oracle import rule as orule

        torch.set_num_threads(os.cpu_count() or 1)
        self.p = problem
        self.lay = orule.Layout.of(problem)
        nq, nk = problem.n_query_tokens, problem.n_key_tokens
        self.rows = np.linspace(0, nq - 1, rows).round().astype(np.int64)
        self.q = W.randn_bf16((nq, heads, W.HEAD_DIM), 1000 * seed).float().numpy()
        self.k = W.randn_bf16((nk, heads, W.HEAD_DIM), 1000 * seed + 1).float().numpy()
        self.v = W.randn_bf16((nk, heads, W.HEAD_DIM), 1000 * seed + 2).float().numpy()
        if int8:   # the cached rows as the INT8 cache holds them (quantised before timing)
            nc = problem.n_cache_tokens
            self.k[:nc] = ocache.dequantize_rows(*ocache.quantize_rows(self.k[:nc]))
            self.v[:nc] = ocache.dequantize_rows(*ocache.quantize_rows(self.v[:nc]))
        self.pairs = sum(sum(b - a for a, b in self.lay.ranges(int(r))) for r in self.rows)
        self.backward = backward
        self.flops = (6.0 if backward else 4.0) * W.HEAD_DIM * heads * self.pairs
        self.desc = (f"oracle (float64 NumPy) on {rows} query rows x {heads} head(s) of "
                     f"{problem.name} ({self.pairs} unmasked pairs per head), as effective "
                     f"TFLOP/s of that sample"
                     + (": the dQ rows (three products per visible pair: S, dP, dS K)"
                        if backward else ""))
        if backward:
            self.d_o = W.randn_bf16((nq, heads, W.HEAD_DIM), 1000 * seed + 3).float().numpy()

    def run(self) -> float:
        from oracle import attention as oattn
        from oracle import backward as obwd

        t0 = time.perf_counter()
        if self.backward:
            obwd.dq_rows(self.lay, self.q, self.k, self.v, self.d_o, self.rows, self.p.softmax_scale)
        else:
            oattn.attention_rows(self.lay, self.q, self.k, self.v, self.rows, self.p.softmax_scale)
        return time.perf_counter() - t0


def camera_bytes(cp) -> int:
    """Algorithmic HBM bytes of one camera cross-attention call: q and x read
    and out written (bf16 [n_q, heads, 128]), the camera K and V read once,
    and the int32 frame index of every query in the frame-aligned modes."""
    row = cp.n_q * cp.heads * W.HEAD_DIM * 2
    return 3 * row + 2 * cp.n_cam * cp.heads * W.HEAD_DIM * 2 + (4 * cp.n_q if cp.mode else 0)


class CameraOracleSample:
    """The camera oracle on `rows` query rows of the workload (every head),
    inputs drawn once; throughput counted in the same algorithmic bytes per
    row as the kernel's."""

    def __init__(self, cp, rows: int, seed: int = 9):
        import numpy as np
        import torch

        torch.set_num_threads(os.cpu_count() or 1)
        self.cp = cp
        rows = min(rows, cp.n_q)
        self.rows = np.linspace(0, cp.n_q - 1, rows).round().astype(np.int64)
        shp = (rows, cp.heads, W.HEAD_DIM)
        self.q = W.randn_bf16(shp, 1000 * seed).float().numpy()
        self.x = W.randn_bf16(shp, 1000 * seed + 1).float().numpy()
        cam = (cp.n_cam, cp.heads, W.HEAD_DIM)
        self.k = W.randn_bf16(cam, 1000 * seed + 2).float().numpy()
        self.v = W.randn_bf16(cam, 1000 * seed + 3).float().numpy()
        self.frame = cp.q_frame()[self.rows]
        self.bytes = camera_bytes(cp) * rows / cp.n_q
        self.desc = (f"oracle (float64 NumPy) on {rows} of the {cp.n_q} query rows x "
                     f"{cp.heads} heads of {cp.name}, as GB/s of the kernel's algorithmic "
                     f"bytes for those rows")

    def run(self) -> float:
        from oracle import camera as ocam

        t0 = time.perf_counter()
        ocam.camera_cross_attention(self.q, self.k, self.v, self.x, self.frame, self.cp.mode,
                                    self.cp.softmax_scale)
        return time.perf_counter() - t0


def cpu_model() -> str:
    """The host CPU's model name (first 'model name' of /proc/cpuinfo)."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.lower().startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def cpu_threads() -> int:
    try:
        import numpy as np  # noqa: F401
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


def run_reference(args, problem):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    if args.workload in CAMERA_WORKLOADS:
        sample = CameraOracleSample(problem, problem.n_q)   # the whole call
        metric, unit = CAMERA_METRIC, "GB/s"
        units = lambda sec: sample.bytes / sec / 1e9  # noqa: E731
        config = {"workload": problem.name, "queries": problem.n_q,
                  "camera_tokens": problem.n_cam, "heads": problem.heads,
                  "head_dim": W.HEAD_DIM, "mode": problem.mode}
    else:
        bwd = args.workload in BWD_WORKLOADS
        sample = OracleSample(problem, args.oracle_rows // (8 if bwd else 1),
                              int8=args.workload in INT8_WORKLOADS, backward=bwd)
        metric, unit = METRIC, "TFLOP/s"
        units = lambda sec: sample.flops / sec / 1e12  # noqa: E731
        config = {"workload": problem.name, "queries": problem.n_query_tokens,
                  "keys": problem.n_key_tokens, "heads": problem.heads, "head_dim": W.HEAD_DIM}
    for _ in range(args.warmup):
        sample.run()
    secs = [sample.run() for _ in range(args.steps)]
    vals = [units(s) for s in secs]
    desc = sample.desc
    config["sample_rows_per_step"] = len(sample.rows)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": metric, "value": value, "unit": unit,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * statistics.mean(secs), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": config,
            "cpu_baseline": {"value": value, "unit": unit, "cores": cpu_threads(),
                             "cpu_model": cpu_model(), "kind": "oracle", "sample": desc},
            "e2e": {"value": value, "unit": unit, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ---------------------------------------------------------------------------
# the native arm
# ---------------------------------------------------------------------------

def reduce_max(x: float, world: int, device: str) -> float:
    """Max of a per-rank number over all ranks (device times are reported as
    the slowest rank's)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tflops(world: int, flops_per_step: float, steps: int, max_ms: float) -> float:
    """Units processed by all ranks divided by the slowest rank's time."""
    return world * flops_per_step * steps / (max_ms * 1e-3) / 1e12


class Session:
    """One replica of the workload on the current device: a cache holding the
    prior segments, the current segment's Q/K/V, outputs and metadata."""

    def __init__(self, problem, seed: int, int8: bool = False, int8_copy: bool = False,
                 nfe: int = 1):
        import torch

        from segment_causal_masked_b200 import sca

        self.sca = sca
        self.p = problem
        dev = torch.device("cuda", torch.cuda.current_device())
        h, nc, nq = problem.heads, problem.n_cache_tokens, problem.n_query_tokens
        self.capacity = (nc + nq + 3) // 4 * 4
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        bf = torch.bfloat16
        self.desc = torch.zeros((self.capacity + 127) // 128 * 128, dtype=torch.int32, device=dev)
        if int8:
            self.k_buf = torch.empty(h, self.capacity, 128, dtype=torch.uint8, device=dev)
            self.v_buf = torch.empty_like(self.k_buf)
            self.k_scale = torch.empty(h, self.capacity, dtype=torch.float32, device=dev)
            self.v_scale = torch.empty_like(self.k_scale)
            self.cache = sca.KVCache(h, self.capacity, self.k_buf, self.v_buf, self.desc,
                                     self.k_scale, self.v_scale)
        else:
            self.k_buf = torch.empty(h, self.capacity, 128, dtype=bf, device=dev)
            self.v_buf = torch.empty_like(self.k_buf)
            self.cache = sca.KVCache(h, self.capacity, self.k_buf, self.v_buf, self.desc)
        self.int8 = int8
        for seg in problem.cached:
            k = torch.randn(seg.n_tokens, h, 128, generator=g, device=dev).to(bf)
            v = torch.randn(seg.n_tokens, h, 128, generator=g, device=dev).to(bf)
            self.cache.append(seg, k, v)
        self.n_prior = len(problem.cached)
        # one current segment = an inference step (append after attention);
        # several = a packed training-shaped forward (no cache append)
        self.appends = len(problem.current) == 1
        # one (Q, K, V) of the current segment per NFE, each drawn afresh
        self.nfe = nfe
        self.qkv = [[torch.randn(nq, h, 128, generator=g, device=dev).to(bf) for _ in range(3)]
                    for _ in range(nfe)]
        self.q, self.k_cur, self.v_cur = self.qkv[0]
        self.outs = [torch.empty(nq, h, 128, dtype=bf, device=dev) for _ in range(nfe)]
        self.o = self.outs[0]
        self.lse = torch.empty(h, nq, dtype=torch.float32, device=dev)
        self.status = torch.zeros(1, dtype=torch.int32, device=dev)
        self.md = sca.build_for(problem)
        ws_bytes = sca.attn_workspace_bytes(self.md, h)
        self.splits = ws_bytes > 0
        if int8_copy:   # room for the bf16 copy of the INT8 cache after the split scratch
            ws_bytes = (ws_bytes + 255) // 256 * 256 + sca.attn_int8_scratch_bytes(self.md, h)
        self.int8_copy = int8_copy
        self.plan = sca.attn_plan(self.md, h)
        self.workspace = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream()
        torch.cuda.synchronize()

    def prepare_backward(self, seed: int):
        """One forward (O, LSE), an upstream gradient dO, gradient outputs and
        the backward's workspace."""
        import torch

        sca, p = self.sca, self.p
        dev = self.q.device
        g = torch.Generator(device=dev)
        g.manual_seed(seed)
        self.md.upload(self.stream.cuda_stream)
        sca.action_causal_attn_fwd(None, self.md, p.heads, self.q, self.k_cur, self.v_cur, self.o,
                                   self.lse, p.softmax_scale, self.workspace, None, self.status,
                                   self.stream.cuda_stream)
        self.d_o = torch.randn(self.q.shape, generator=g, device=dev).to(torch.bfloat16)
        self.dq, self.dk, self.dv = (torch.empty_like(self.q) for _ in range(3))
        self.bws = torch.empty(sca.attn_bwd_workspace_bytes(self.md, p.heads), dtype=torch.uint8,
                               device=dev)
        torch.cuda.synchronize()

    def step_backward(self, q=None, k=None, v=None, o=None, lse=None, d_o=None, grads=None,
                      ev=None):
        """One backward call; `grads` = (dq, dk, dv) outputs (the session's by
        default); `ev` = (start, end) events around it."""
        sca, p = self.sca, self.p
        s = self.stream.cuda_stream
        dq, dk, dv = grads if grads is not None else (self.dq, self.dk, self.dv)
        if ev is not None:
            ev[0].record(self.stream)
        sca.action_causal_attn_bwd(self.md, p.heads, self.q if q is None else q,
                                   self.k_cur if k is None else k, self.v_cur if v is None else v,
                                   self.o if o is None else o, self.lse if lse is None else lse,
                                   self.d_o if d_o is None else d_o, dq, dk, dv,
                                   p.softmax_scale, self.bws, None, self.status, s)
        if ev is not None:
            ev[1].record(self.stream)

    def step(self, ins=None, outs=None, ev=None):
        """One pass of the hot path: the metadata built and uploaded, one
        attention call per NFE, then the append. ``ins`` = [q, k_cur, v_cur]
        per NFE and ``outs`` = [o] per NFE (the session's own by default);
        ``ev`` = one (start, end) event pair per attention call."""
        sca, p = self.sca, self.p
        s = self.stream.cuda_stream
        sca.build_for(p, self.md)
        self.md.upload(s)
        qkv = self.qkv if ins is None else [ins[3 * i:3 * i + 3] for i in range(self.nfe)]
        outs = self.outs if outs is None else outs
        for i in range(self.nfe):
            q, k_cur, v_cur = qkv[i]
            if ev is not None:
                ev[i][0].record(self.stream)
            sca.action_causal_attn_fwd(self.cache, self.md, p.heads, q, k_cur, v_cur, outs[i],
                                       self.lse, p.softmax_scale, self.workspace, None,
                                       self.status, s)
            if ev is not None:
                ev[i][1].record(self.stream)
        if self.appends:  # inference: the generated segment joins the cache
            self.cache.append(p.current[0], qkv[-1][1], qkv[-1][2], s)
            self.cache.truncate(self.n_prior)


def init_ranks(args):
    """(world, rank, local rank) from the torchrun environment; the device
    set and, for N > 1, the NCCL process group up (used for the barrier and
    the max over ranks only)."""
    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}; launch N>1 with torchrun")
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    return world, rank, local


def run_native(args, problem):
    import torch
    import torch.distributed as dist

    world, rank, local = init_ranks(args)

    def barrier():
        if world > 1:
            dist.barrier()

    def max_over_ranks(x: float) -> float:
        return reduce_max(x, world, "cuda")

    int8 = args.workload in INT8_WORKLOADS
    bwd = args.workload in BWD_WORKLOADS
    int8_copy = args.workload in INT8_COPY_WORKLOADS
    nfe = NFE_WORKLOADS.get(args.workload, 1)
    sess = Session(problem, seed=1000 * 2 + rank, int8=int8, int8_copy=int8_copy, nfe=nfe)
    from segment_causal_masked_b200 import sca
    sca_md = sca.build_for(problem)
    counts = sca_md.counts()
    A = counts["unmasked_pairs"]
    flops_call = effective_flops(problem, A)   # one attention call (one NFE)
    flops = nfe * flops_call                     # one step
    step = sess.step
    if bwd:
        sess.prepare_backward(1000 * 3 + rank)
        flops *= BWD_FLOP_FACTOR
        flops_call = flops
        step = sess.step_backward

    # ---- device-resident timing
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    # one (start, end) pair around every attention call (the backward: the call)
    evs = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(1 if bwd else nfe)] for _ in range(args.steps)]
    t_start, t_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t_start.record(sess.stream)
    for i in range(args.steps):
        step(ev=evs[i][0] if bwd else evs[i])
    t_end.record(sess.stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier()
    if int(sess.status.item()) != 0:
        raise SystemExit(f"device status {int(sess.status.item())}")
    ms_total = max_over_ranks(t_start.elapsed_time(t_end))
    attn_ms = [a.elapsed_time(b) for calls in evs for a, b in calls]
    attn_avg = max_over_ranks(statistics.mean(attn_ms))
    ms_step = ms_total / args.steps
    value = whole_job_tflops(world, flops, args.steps, ms_total)

    # ---- end to end through the API with pinned host buffers. Every step
    # uploads its inputs from pinned host memory and downloads its result;
    # with two device copies of the inputs and outputs, step i+1's uploads
    # (one stream) and step i's download (another) overlap step i's compute,
    # as a serving loop would run. All of it lies inside the timed region.
    nq, h = problem.n_query_tokens, problem.heads
    pin = dict(pin_memory=True, dtype=torch.bfloat16)
    if bwd:   # inputs q, k, v, o, lse, dO; results dq, dk, dv
        host_in = [t.cpu().pin_memory() for t in (sess.q, sess.k_cur, sess.v_cur, sess.o, sess.lse,
                                                  sess.d_o)]
        host_out = [torch.empty(nq, h, 128, **pin) for _ in range(3)]

        def run(ins, outs):
            q, k, v, o, lse, d_o = ins
            sess.step_backward(q=q, k=k, v=v, o=o, lse=lse, d_o=d_o, grads=outs)
    else:     # inputs q, k_cur, v_cur of every NFE; result o of every NFE
        host_in = [t.cpu().pin_memory() for qkv in sess.qkv for t in qkv]
        host_out = [torch.empty(nq, h, 128, **pin) for _ in range(nfe)]

        def run(ins, outs):
            sess.step(ins=ins, outs=outs)
    dev_in = [[torch.empty_like(t, device="cuda") for t in host_in] for _ in range(2)]
    dev_out = [[torch.empty_like(t, device="cuda") for t in host_out] for _ in range(2)]
    bytes_in = sum(t.numel() * t.element_size() for t in host_in)
    bytes_out = sum(t.numel() * t.element_size() for t in host_out)
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, out_ready, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [None, None]   # event after the compute that last read input set b

    def upload(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            if used[b] is not None:
                h2d.wait_event(used[b])
            for dst, src in zip(dev_in[b], host_in):
                dst.copy_(src, non_blocking=True)
            in_ready[b].record(h2d)

    def e2e_steps(n):
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            sess.stream.wait_event(in_ready[b])
            sess.stream.wait_event(out_read[b])
            run(dev_in[b], dev_out[b])
            used[b] = ev()
            used[b].record(sess.stream)
            out_ready[b].record(sess.stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(out_ready[b])
                for dst, src in zip(host_out, dev_out[b]):
                    dst.copy_(src, non_blocking=True)
                out_read[b].record(d2h)
        last = ev()
        last.record(d2h)
        sess.stream.wait_event(last)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(sess.stream)
    h2d.wait_event(e0)
    e2e_steps(args.steps)
    e1.record(sess.stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = whole_job_tflops(world, flops, args.steps, e2e_ms)

    if rank == 0:
        peaks = measured_peaks()
        sustained = attn_avg >= SUSTAINED_CALL_MS
        peak = float(peaks["bf16_tflops_sustained" if sustained else "bf16_tflops"])
        achieved = flops_call / (attn_avg * 1e-3) / 1e12
        traffic = None if bwd else stored_traffic("attn_fwd_kernel", problem.name)
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": problem.name, "queries": nq, "keys": problem.n_key_tokens,
                       "cached_segments": len(problem.cached), "heads": h,
                       "head_dim": W.HEAD_DIM, "unmasked_pairs_per_head": A,
                       "effective_flop_per_step": flops,
                       "step": ("attention backward (D and LSE, dQ, dK and dV kernels); the "
                                "forward that produced O and LSE ran once before timing" if bwd
                                else ("metadata build+upload, %d attention forwards (one per "
                                      "NFE, each with its own current-segment Q, K, V), "
                                      "kv_cache_append" % nfe) if nfe > 1
                                else "metadata build+upload, attention forward, kv_cache_append"
                                if sess.appends else "metadata build+upload, attention forward"),
                       "nfe": nfe,
                       "flop_count": ("10·d·H·A (five products per visible pair)" if bwd
                                      else "4·d·H·A (two products per visible pair)"
                                      + (" per NFE" if nfe > 1 else "")),
                       "kv_cache": ("int8 codes + fp32 row scales" + (", dequantised once per call"
                                    " into a bf16 copy in the workspace" if int8_copy else
                                    ", dequantised tile by tile in the kernel")) if int8 else "bf16",
                       "l2": "inputs larger than L2 (cached K/V %.2f GB per tensor)"
                             % (problem.n_cache_tokens * h * (132 if int8 else 256) / 1e9),
                       "parallelism": f"replicas x{world}",
                       "split_plan": sess.plan},
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak,
                         "unit": "TFLOP/s", "frac": achieved / peak, "traffic": traffic,
                         "kernel": ("bwd_prep_kernel + bwd_dq_kernel + bwd_dkdv_kernel" if bwd
                                    else "attn_fwd_kernel"), "kernel_ms": attn_avg,
                         "kernel_ms_is": ("per backward call" if bwd else
                                          "per attention call (one NFE)"),
                         "peak_source": f"{peaks['source']} bf16 dense "
                                        + ("(sustained: the call lasts over %.1f s)"
                                           % (SUSTAINED_CALL_MS / 1e3) if sustained
                                           else "(burst)")},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": bytes_in,
                    "d2h_bytes_per_step": bytes_out, "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": (3 if bwd else nfe * (1 + int(sess.splits) + int(int8_copy))
                             + int(sess.appends)) * args.steps,
            "clocks": clock_info,
        }
        if not args.no_cpu_baseline:
            sample = OracleSample(problem, args.baseline_rows // (8 if bwd else 1), int8=int8,
                                  backward=bwd)
            dt = sample.run()
            line["cpu_baseline"] = {"value": sample.flops / dt / 1e12, "unit": "TFLOP/s",
                                    "cores": cpu_threads(), "cpu_model": cpu_model(),
                                    "kind": "oracle", "sample": sample.desc, "seconds": dt}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_camera(args, cp):
    """The camera cross-attention call of one segment: K calls timed on the
    device as one CUDA-graph replay (inputs rotated over CAMERA_INPUT_SETS
    sets, larger than L2 together), and end to end through the API, eagerly,
    with every step's inputs uploaded from and its output read back to pinned
    host memory."""
    import torch
    import torch.distributed as dist

    from segment_causal_masked_b200 import sca

    world, rank, local = init_ranks(args)
    dev = torch.device("cuda", local)
    g = torch.Generator(device=dev)
    g.manual_seed(1000 * 5 + rank)
    bf = torch.bfloat16
    shp, cam = (cp.n_q, cp.heads, W.HEAD_DIM), (cp.n_cam, cp.heads, W.HEAD_DIM)
    sets = [[torch.randn(shp, generator=g, device=dev).to(bf) for _ in range(3)]
            for _ in range(CAMERA_INPUT_SETS)]   # q, x, out
    k_cam = torch.randn(cam, generator=g, device=dev).to(bf)
    v_cam = torch.randn(cam, generator=g, device=dev).to(bf)
    frame = torch.from_numpy(cp.q_frame()).to(dev)
    stream = torch.cuda.current_stream()
    status = torch.zeros(1, dtype=torch.int32, device=dev)

    def call(q, x, out, fr, kc, vc):
        sca.camera_cross_attn(q, kc, vc, x, out, fr, cp.mode, cp.softmax_scale,
                              dev_status=status,
                              stream=torch.cuda.current_stream().cuda_stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for i in range(args.warmup):
        q, x, out = sets[i % CAMERA_INPUT_SETS]
        call(q, x, out, frame, k_cam, v_cam)
    torch.cuda.synchronize()
    # Device-resident timing. One call takes less device time than the host
    # needs to encode its tensor maps and launch it, so back-to-back calls
    # from the host would time the host: the K calls are captured once as a
    # CUDA graph (the same launches, each with its own tensor maps) and the
    # replay is timed.
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, capture_error_mode="relaxed"):
        for i in range(args.steps):
            q, x, out = sets[i % CAMERA_INPUT_SETS]
            call(q, x, out, frame, k_cam, v_cam)
    graph.replay()   # one untimed replay
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local)
    barrier()
    torch.cuda.synchronize()
    clocks.start()
    t0.record(stream)
    graph.replay()
    t1.record(stream)
    torch.cuda.synchronize()
    clock_info = clocks.stop()
    barrier()
    if int(status.item()) != 0:
        raise SystemExit(f"device status {int(status.item())}")
    nbytes = camera_bytes(cp)
    ms_total = reduce_max(t0.elapsed_time(t1), world, "cuda")
    call_ms = ms_total / args.steps
    value = world * nbytes * args.steps / (ms_total * 1e-3) / 1e9
    del graph

    # end to end: q, x, the frames and the camera K/V uploaded from pinned
    # host memory, the call, out read back; uploads of step i+1 (one stream)
    # and the read-back of step i (another) overlap step i's call
    host_in = [t.cpu().pin_memory() for t in (sets[0][0], sets[0][1], frame, k_cam, v_cam)]
    host_out = torch.empty(shp, dtype=bf, pin_memory=True)
    dev_in = [[torch.empty_like(t, device=dev) for t in host_in] for _ in range(2)]
    dev_out = [torch.empty(shp, dtype=bf, device=dev) for _ in range(2)]
    bytes_in = sum(t.numel() * t.element_size() for t in host_in)
    bytes_out = host_out.numel() * host_out.element_size()
    h2d, d2h = torch.cuda.Stream(), torch.cuda.Stream()
    ev = torch.cuda.Event
    in_ready, out_ready, out_read = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    used = [None, None]

    def upload(i):
        b = i % 2
        with torch.cuda.stream(h2d):
            if used[b] is not None:
                h2d.wait_event(used[b])
            for dst, src in zip(dev_in[b], host_in):
                dst.copy_(src, non_blocking=True)
            in_ready[b].record(h2d)

    def e2e_steps(n):
        upload(0)
        for i in range(n):
            b = i % 2
            if i + 1 < n:
                upload(i + 1)
            stream.wait_event(in_ready[b])
            stream.wait_event(out_read[b])
            q, x, fr, kc, vc = dev_in[b]
            call(q, x, dev_out[b], fr, kc, vc)
            used[b] = ev()
            used[b].record(stream)
            out_ready[b].record(stream)
            with torch.cuda.stream(d2h):
                d2h.wait_event(out_ready[b])
                host_out.copy_(dev_out[b], non_blocking=True)
                out_read[b].record(d2h)
        last = ev()
        last.record(d2h)
        stream.wait_event(last)

    e2e_steps(args.warmup)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    e0.record(stream)
    h2d.wait_event(e0)
    e2e_steps(args.steps)
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = reduce_max(e0.elapsed_time(e1), world, "cuda")
    e2e_value = world * nbytes * args.steps / (e2e_ms * 1e-3) / 1e9

    if rank == 0:
        peaks = measured_peaks()
        peak = float(peaks["hbm_gbs"])
        achieved = nbytes / (call_ms * 1e-3) / 1e9
        traffic = stored_traffic("camera_xattn_kernel", cp.name)
        line = {
            "metric": CAMERA_METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_total / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": cp.name, "queries": cp.n_q, "camera_tokens": cp.n_cam,
                       "heads": cp.heads, "head_dim": W.HEAD_DIM, "mode": cp.mode,
                       "algorithmic_bytes_per_step": nbytes,
                       "step": "one camera cross-attention call (out = x + attention)",
                       "l2": "q, x, out rotated over %d sets (%.0f MB together) > L2"
                             % (CAMERA_INPUT_SETS, CAMERA_INPUT_SETS * 3 * cp.n_q * cp.heads
                                * W.HEAD_DIM * 2 / 1e6),
                       "parallelism": f"replicas x{world}"},
            "pct_of_peak": 100.0 * value / world / peak,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "kernel": "camera_xattn_kernel", "kernel_ms": call_ms,
                         "kernel_ms_is": "graph replay of the K calls / K (one kernel per call)",
                         "peak_source": f"{peaks['source']} HBM copy bandwidth"},
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": bytes_in,
                    "d2h_bytes_per_step": bytes_out, "ms_per_step": e2e_ms / args.steps},
            "gpu_launches": args.steps,
            "clocks": clock_info,
        }
        if not args.no_cpu_baseline:
            sample = CameraOracleSample(cp, cp.n_q)   # the whole call
            dt = sample.run()
            line["cpu_baseline"] = {"value": sample.bytes / dt / 1e9, "unit": "GB/s",
                                    "cores": cpu_threads(), "cpu_model": cpu_model(),
                                    "kind": "oracle", "sample": sample.desc, "seconds": dt}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--workload", choices=sorted(WORKLOADS), default="480p-long-session")
    ap.add_argument("--oracle-rows", type=int, default=384,
                    help="query rows per step of the reference arm")
    ap.add_argument("--baseline-rows", type=int, default=8192,
                    help="query rows of the cpu_baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)   # at least 3 untimed warm-up steps
    problem = WORKLOADS[args.workload]()
    if args.impl == "reference":
        return run_reference(args, problem)
    if args.workload in CAMERA_WORKLOADS:
        return run_camera(args, problem)
    return run_native(args, problem)


if __name__ == "__main__":
    sys.exit(main())
