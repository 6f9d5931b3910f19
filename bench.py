"""Throughput of the ARL2 hybrid attention layer: frames/s per layer at the 480p workload.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one autoregressive frame of one layer: 4 denoising queries (intra-frame softmax
attention plus the state readout) and the clean-pass commit of the state. This is every
step of the layer's hot path.

The workload is 480p: B=1, H=12, d=128, T=1560 tokens per frame. Inputs are seeded and
synthetic (q, k, v ~ N(0,1) in bf16; phi ~ N(0, 1/d); alpha = sigmoid(N(2, 0.5));
beta = sigmoid(N(0,1))). The timed region cycles through 8 frames of distinct inputs,
5 passes per frame (4 denoising + 1 clean), about 575 MB. That is larger than the 126 MB
L2, so no input is L2-resident between frames.

The bench prints one JSON line (rank 0):
  - value: whole-job frames/s, timed on the device with CUDA events between barriers.
  - e2e: the same metric through the host-buffer entry points. Each step copies its
    inputs from pinned host memory and its outputs back.
  - repeats: the same timed window of K frames, repeated; median and spread of frames/s.
  - roofline: the query kernel's achieved TFLOP/s (algorithmic FLOPs / mean launch time,
    CUDA events on the launching stream, from a second timed region that runs windows of
    queries back to back, then commits back to back, with launch overlap off) against the
    measured bf16 burst peak (the kernel is timed on its own, not inside a long mixed step).
    roofline_commit: the commit's achieved GB/s (algorithmic bytes / mean launch time,
    timed the same way) against the measured HBM copy bandwidth.
  Every device-timed region starts behind a spin kernel queued ahead of its first event, so
  its launches run back to back and its events measure device time, not Python's launch
  rate (the host-buffer e2e leg has no such spin: it measures the host too).
  - frame_roofline: the whole frame (4 queries + 1 commit, overlapped) against both peaks.
  - stream: 240 frames, each bracketed by events: per-frame time first/last and its slope,
    and device memory (cudaMemGetInfo) before and after.
  - sweep: frames/s and the two kernels' roofline fractions at B in {1, 4} and
    T in {390, 1560, 3600} (device-generated seeded inputs, larger than L2 per cycle).
  - hybrid_stack: timing-only 30-layer stacks with 0%, 50% and 75% of the layers ARL2 and
    the rest softmax over a growing KV cache: time per frame and N-dependent memory at
    frame N = 1, 21, 60, 120.
  - token_level: the token-level access ablation (4 queries + 1 commit per frame, each call
    alone), its scan against the SMs' fp32 rate.
  - clean_pass: frames with the fused clean pass (4 queries + clean pass) against frames with
    its two calls (4 queries + query + commit), and the clean pass alone against the pair.
  - cpu_baseline: the fp64 oracle on this host's cores over a bounded sample.
  - clocks: SM clocks and throttle reasons sampled with NVML during the timed region.
With --gpus N under torchrun, each rank runs its own independent layer (the layer has no
exchange between streams: replicas, weak scaling).
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

from softmax_attention_ar_b200 import synth  # noqa: E402

WORKLOAD = synth.WORKLOADS["480p"]
B, T, H, D = WORKLOAD["B"], WORKLOAD["T"], WORKLOAD["H"], WORKLOAD["d"]
QUERIES = WORKLOAD["queries"]
CYCLE = 8                      # distinct frames of inputs in the timed cycle
METRIC = "frames/s per ARL2 layer at T=1560,H=12,d=128; % bf16 TC peak & % HBM BW"
UNIT = "frames/s"
CONFIG = {"workload": "480p single layer: B=1, H=12, d=128, T=1560 tokens/frame; "
                      "4 denoising queries + 1 clean-pass commit per frame",
          "B": B, "H": H, "T": T, "d": D, "queries_per_frame": QUERIES,
          "l2": "inputs larger than L2 (8-frame cycle of distinct q/k/v, 575 MB)"}

# Algorithmic work (only what the layer must do; padding of ragged tiles is not credited).
def query_flops(b, t, h, d):      # QK^T + PV, phi_q + readout
    return b * h * (4.0 * t * t * d + 2 * 2.0 * t * d * d)


def query_bytes(b, t, h, d):      # q, k, v, o bf16; S bf16 copy, Wq
    return b * t * h * d * 2 * 4 + b * h * d * d * (2 + 2)


def commit_flops(b, t, h, d):     # K Wk, V Wv, K'S, K'^T R
    return b * h * 4 * 2.0 * t * d * d


def commit_bytes(b, t, h, d):     # k, v bf16; alpha, beta; S read + write fp32; Wk, Wv
    return b * t * h * d * 2 * 2 + 2 * b * h * t * 4 + b * h * d * d * 4 * 2 + 2 * h * d * d * 2


QUERY_FLOPS, QUERY_BYTES = query_flops(B, T, H, D), query_bytes(B, T, H, D)
COMMIT_FLOPS, COMMIT_BYTES = commit_flops(B, T, H, D), commit_bytes(B, T, H, D)
FRAME_FLOPS = QUERIES * QUERY_FLOPS + COMMIT_FLOPS
FRAME_BYTES = QUERIES * QUERY_BYTES + COMMIT_BYTES


# NVIDIA's dense (no 2:4 sparsity) bf16 tensor-core figure for one B200, for context only; the
# roofline fraction uses the measured peak.
DATASHEET_BF16_TFLOPS = 2250.0


KERNEL_HEADERS = {"arl2_query.cu": ("arl2_query_body.cuh",)}


def kernel_sources_sha256(kernel_file: str) -> str:
    """SHA-256 over a kernel's source file and the headers it includes."""
    import hashlib
    csrc = os.path.join(ROOT, "softmax_attention_ar_b200", "csrc")
    digest = hashlib.sha256()
    for f in (kernel_file, *KERNEL_HEADERS.get(kernel_file, ()), "arl2_device.cuh", "arl2_kernels.h"):
        with open(os.path.join(csrc, f), "rb") as fh:
            digest.update(fh.read())
    return digest.hexdigest()


def _profile_traffic(summary: str, kernel_file: str):
    """DRAM bytes per launch from a committed ncu summary, or None when the kernel's sources
    changed since that capture (the summary records their SHA-256)."""
    import re
    path = os.path.join(ROOT, "profiles", summary)
    if not os.path.exists(path):
        return None
    text = open(path).read()
    t = re.search(r"^traffic_bytes_per_launch: (\d+)$", text, re.M)
    h = re.search(r"^kernel_sources_sha256: ([0-9a-f]{64})$", text, re.M)
    if not t or not h:
        return None
    return int(t.group(1)) if kernel_sources_sha256(kernel_file) == h.group(1) else None


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML (read-only) in a thread."""

    REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap", 0x8: "hw_slowdown",
               0x10: "sync_boost", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x100: "display_clock_setting"}

    def __init__(self, index: int):
        self.samples, self.reasons, self._stop = [], set(), threading.Event()
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self._nv = None

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                self.reasons.update(n for b, n in self.REASONS.items() if mask & b)
            except Exception:
                pass
            self._stop.wait(0.02)

    def __enter__(self):
        if self._nv is not None:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._nv is not None:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons - {"gpu_idle"}), "samples": len(self.samples)}


def make_inputs(dev):
    import torch

    def bf(x):
        return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)

    frames = []
    for f in range(CYCLE):
        passes = [tuple(bf(x) for x in synth.qkv(0, WORKLOAD["config"], f, p, B, T, H, D))
                  for p in range(QUERIES + 1)]
        a, b = synth.gates(0, WORKLOAD["config"], f, B, H, T)
        frames.append((passes, torch.from_numpy(a), torch.from_numpy(b)))
    wq, wk, wv = (bf(x) for x in synth.feature_maps(0, WORKLOAD["config"], H, D))
    if dev is None:
        return frames, (wq, wk, wv)
    dev_frames = [([tuple(t.to(dev) for t in p) for p in passes], a.to(dev), b.to(dev)) for passes, a, b in frames]
    return dev_frames, (wq.to(dev), wk.to(dev), wv.to(dev)), frames


class OracleSample:
    """A bounded slice of one 480p frame for the fp64 oracle: the 4 queries of one head on R
    query rows, and that head's commit over R tokens. Work grows linearly in R, so the slice
    stands for R / (T * H) of a frame."""

    def __init__(self):
        import oracle
        self.oracle = oracle
        cfg = WORKLOAD["config"]
        wq, wk, wv = (synth.bf16_to_f64(x)[:1] for x in synth.feature_maps(0, cfg, H, D))
        self.W = (wq, wk, wv)
        self.passes = [tuple(synth.bf16_to_f64(x)[:, :, :1] for x in synth.qkv(0, cfg, 0, p, B, T, H, D))
                       for p in range(QUERIES + 1)]
        a, b = synth.gates(0, cfg, 0, B, H, T)
        self.gates = (a[:, :1], b[:, :1])
        self.S = np.zeros((B, 1, D, D))

    def run(self, R: int) -> float:
        """Run one slice; return the fraction of a frame it stands for."""
        rows = np.arange(R)
        for p in range(QUERIES):
            self.oracle.frame_query(*self.passes[p], self.W[0], self.S, rows=rows)
        _, k, v = self.passes[QUERIES]
        self.S = self.oracle.frame_commit(k[:, :R], v[:, :R], self.gates[0][..., :R], self.gates[1][..., :R],
                                          self.W[1], self.W[2], self.S)
        return R / (T * H)


def _oracle_rate(steps: int, warmup: int, budget_s: float):
    """Time `steps` oracle slices sized so the run takes about budget_s; return (frames/s, R, seconds)."""
    from threadpoolctl import threadpool_info
    s = OracleSample()
    t0 = time.perf_counter()
    s.run(T)                                  # calibrate on one full head
    full = time.perf_counter() - t0
    R = int(max(8, min(T, T * budget_s / max(1, steps + warmup) / full)))
    for _ in range(warmup):
        s.run(R)
    t0 = time.perf_counter()
    frac = sum(s.run(R) for _ in range(steps))
    dt = time.perf_counter() - t0
    threads = max([i.get("num_threads", 1) for i in threadpool_info()] or [1])
    return frac / dt, R, dt, threads


def cpu_baseline(budget_s: float = 15.0):
    """The fp64 oracle, as it stands, on this host's cores: frames/s over a bounded sample."""
    steps = 12
    rate, R, dt, threads = _oracle_rate(steps, 1, budget_s)
    return {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{steps} slices of a 480p frame, each the 4 queries of one head on {R} of {T} query rows "
                      f"plus that head's commit over {R} tokens ({steps * R / (T * H):.3f} frames in {dt:.1f} s); "
                      f"fp64 numpy/BLAS, {os.cpu_count()} host cores"}


def kv_cache_baseline(frames, dev, layer_ms_per_frame, layer_bytes):
    """The growing-KV-cache baseline the layer replaces (softmax attention of the newest frame
    over every cached frame), on the same seeded q, k, v: time for the 4 queries of frame N
    (CUDA events, mean of 3) and its KV memory, at N = 21, 60 and 120 cached frames."""
    import torch

    from softmax_attention_ar_b200.arl2 import KVCacheBaseline
    Ns = (21, 60, 120)
    base = KVCacheBaseline(H, T, D, B, max_frames=max(Ns))
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    stream = torch.cuda.current_stream()
    frame_kv = B * T * H * D * 2 * 2
    rows = []
    for N in Ns:
        base.reset()
        for f in range(N - 1):
            _, k, v = frames[f % CYCLE][0][QUERIES][:3]
            base.commit(k, v)
        passes = [p[:3] for p in frames[(N - 1) % CYCLE][0]]
        for p in range(QUERIES):                       # warm-up
            base.query(*passes[p], out=o)
        st, en = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        st.record(stream)
        for _ in range(3):
            for p in range(QUERIES):
                base.query(*passes[p], out=o)
        en.record(stream)
        torch.cuda.synchronize()
        rows.append({"N": N, "queries_ms_per_frame": st.elapsed_time(en) / 3, "kv_bytes": N * frame_kv})
    status = base.status()
    allocated = base.memory_bytes
    base.close()
    return {"what": "softmax attention of each frame's 4 queries over all N cached frames (growing KV cache), "
                    "same kernel main loop; time excludes the cache appends",
            "frames": rows, "allocated_bytes": allocated, "status": status,
            "arl2_ms_per_frame": layer_ms_per_frame, "arl2_state_bytes": layer_bytes}


def hybrid_stack(frames, dev, stream, layers=30, Ns=(1, 21, 60, 120), shares=(0.0, 0.5, 0.75)):
    """Timing-only stack of `layers` attention layers at the 480p shapes: a share of them ARL2
    layers, the rest softmax attention over a growing KV cache (the layers ARL2 replaces). For
    frame N: the time of one frame of the whole stack (per layer its 4 denoising queries and
    the clean pass's commit, or cache append), CUDA events over two consecutive frames, and
    the device memory that depends on N (the KV caches; each ARL2 layer's state is constant).
    Synthetic weights and inputs: this reproduces the shape of the memory and time curves with
    video length, not any model's quality."""
    import torch

    from softmax_attention_ar_b200.arl2 import ARL2Layer, KVCacheBaseline
    Nmax = max(Ns) + 2
    frame_kv = B * T * H * D * 2 * 2                 # one frame's K and V, bf16
    n_soft_max = max(layers - int(round(s * layers)) for s in shares)
    n_arl2_max = max(int(round(s * layers)) for s in shares)
    caches = [KVCacheBaseline(H, T, D, B, max_frames=Nmax) for _ in range(n_soft_max)]
    arl2s = [ARL2Layer(H, T, D, B) for _ in range(n_arl2_max)]
    wq = torch.randn((H, D, D), device=dev, dtype=torch.float32).div_(D ** 0.5).to(torch.bfloat16)
    for lay in arl2s:
        lay.set_feature_maps(wq, wq, wq)
        lay.set_launch_overlap(True)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    state_bytes = B * H * D * D * (4 + 4 + 2 + 2)    # fp32 state, its other buffer and their bf16 copies
    out = {"layers": layers, "what": "timing-only: 4 queries + 1 commit (or cache append) per layer per frame; "
                                     "softmax layers attend over every cached frame plus the current one",
           "kv_bytes_per_frame_per_softmax_layer": frame_kv, "arl2_state_bytes_per_layer": state_bytes, "shares": {}}
    for share in shares:
        n_arl2 = int(round(share * layers))
        n_soft = layers - n_arl2
        rows = []
        for N in Ns:
            for c in caches[:n_soft]:
                c.reset()
                for f in range(N - 1):
                    _, k, v = frames[f % CYCLE][0][QUERIES][:3]
                    c.commit(k, v)
            for lay in arl2s[:n_arl2]:
                lay.reset()

            def stack_frame(f, mid=None):
                passes, a, b = frames[f % CYCLE]
                for i in range(layers):
                    if i == n_arl2 and mid is not None:
                        mid.record(stream)   # the ARL2 layers are done, the softmax layers start
                    if i < n_arl2:      # ARL2 layers first; order does not change the total
                        lay = arl2s[i]
                        for p in range(QUERIES):
                            lay.query(*passes[p][:3], out=o)
                        _, k, v = passes[QUERIES][:3]
                        lay.commit(k, v, a, b)
                    else:
                        c = caches[i - n_arl2]
                        for p in range(QUERIES):
                            c.query(*passes[p][:3], out=o)
                        _, k, v = passes[QUERIES][:3]
                        c.commit(k, v)

            torch.cuda.synchronize()
            # A softmax layer's query also copies the frame's k and v into the cache: count
            # every copy as a launch.
            queue_ahead(2 * (n_arl2 * (QUERIES + 1) + n_soft * (3 * QUERIES + 2)) + 2)
            st, md, mid, en = (torch.cuda.Event(enable_timing=True) for _ in range(4))
            st.record(stream)
            stack_frame(N - 1)
            md.record(stream)
            stack_frame(N, mid)
            en.record(stream)
            torch.cuda.synchronize()
            row = {"N": N, "ms_per_frame": st.elapsed_time(en) / 2, "kv_bytes": n_soft * N * frame_kv,
                   "arl2_state_bytes": n_arl2 * state_bytes}
            if 0 < n_arl2 < layers:   # the second frame split at the last ARL2 layer
                row["ms_arl2_layers"] = md.elapsed_time(mid)
                row["ms_softmax_layers"] = mid.elapsed_time(en)
            rows.append(row)
        out["shares"][f"{share:.2f}"] = {"arl2_layers": n_arl2, "softmax_layers": n_soft, "frames": rows}
    status = [c.status() for c in caches] + [lay.status() for lay in arl2s]
    out["status"] = max(status) if status else 0
    for c in caches:
        c.close()
    for lay in arl2s:
        lay.close()
    torch.cuda.empty_cache()
    return out


def max_over_ranks(values, device, world):
    """Each rank's timings -> the maximum over ranks, elementwise (the job is as slow as its
    slowest rank). Uses the default process group when world > 1."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def job_rate(world, frames_per_rank, elapsed_ms):
    """Whole-job frames/s: every rank's frames over the slowest rank's time."""
    return world * frames_per_rank / (elapsed_ms / 1e3)


def run_reference(args, rank, world):
    """Reference arm: the fp64 oracle on the host cores, same metric and workload."""
    if rank != 0:
        return
    rate, R, dt, threads = _oracle_rate(args.steps, args.warmup, budget_s=90.0)
    base = {"value": rate, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"each step: the 4 queries of one head on {R} of {T} query rows plus that head's commit "
                      f"over {R} tokens (= {R / (T * H):.5f} frame)"}
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * dt / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": CONFIG, "cpu_baseline": base,
            "e2e": {"value": rate, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# fp32 FMA rate of the SMs (no tensor cores): 148 SMs x 128 lanes x 2 flops x 1.965 GHz.
FP32_PEAK_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12
HOST_MS_PER_LAUNCH = 0.05   # generous bound on the host's cost to enqueue one launch or event


def queue_ahead(launches: int):
    """Keep the device busy while the host enqueues the next timed region: a spin kernel
    (torch.cuda._sleep) long enough for the host to queue `launches` launches behind it, so
    the region's launches run back to back and its events measure device time only, not the
    host's enqueue rate. Goes on the current stream before the region's first event."""
    import torch
    torch.cuda._sleep(int(2.0e6 * (0.5 + HOST_MS_PER_LAUNCH * launches)))   # ~2e6 cycles per ms


def _time_windows(run_frame, stream, n_windows, frames_per_window, start, barrier):
    """n_windows back-to-back windows of frames_per_window frames; each window bracketed by
    CUDA events on the launching stream. Returns the frames/s of each window."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_windows)]
    barrier()
    queue_ahead(n_windows * frames_per_window * (QUERIES + 1) + 2 * n_windows)
    i = start
    for s, e in evs:
        s.record(stream)
        for _ in range(frames_per_window):
            run_frame(i)
            i += 1
        e.record(stream)
    barrier()
    return [frames_per_window / (s.elapsed_time(e) / 1e3) for s, e in evs]


def _split_times(layer, frames, stream, n, barrier, queries=QUERIES, window=10):
    """Per-kernel split, overlap off: windows of `window` frames, each running its 4 x window
    queries back to back between one pair of events, then its `window` commits back to back
    between another. A window's time / its launches is one sample of that kernel's average
    launch duration in a stream (kernel time plus the gap between queued launches; no event
    sits between two launches). Returns (query samples in ms, commit samples in ms)."""
    import torch
    layer.set_launch_overlap(False)
    nw = max(1, n // window)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(nw)]
    barrier()
    queue_ahead(nw * (window * (queries + 1) + 4))
    for w in range(nw):
        idx = [(w * window + i) % len(frames) for i in range(window)]
        ev[w][0].record(stream)
        for i in idx:
            passes = frames[i][0]
            for p in range(queries):
                layer.query(*passes[p][:3], out=passes[p][3])
        ev[w][1].record(stream)
        ev[w][2].record(stream)
        for i in idx:
            passes, a, b = frames[i]
            _, k, v, _ = passes[queries]
            layer.commit(k, v, a, b)
        ev[w][3].record(stream)
    barrier()
    q_ms = [e[0].elapsed_time(e[1]) / (window * queries) for e in ev]
    c_ms = [e[2].elapsed_time(e[3]) / window for e in ev]
    return q_ms, c_ms


def _rooflines(q_ms, c_ms, b, t, h, d, peaks):
    """Achieved rates of the two kernels (per-launch averages of back-to-back launches of one
    kind, overlap off) against the burst peaks; p95 is over the timing windows."""
    q_s, c_s = statistics.mean(q_ms) / 1e3, statistics.mean(c_ms) / 1e3
    q_tf = query_flops(b, t, h, d) / q_s / 1e12
    c_gbs = commit_bytes(b, t, h, d) / c_s / 1e9
    return {"query_us": 1e6 * q_s, "query_p95_us": 1e3 * float(np.percentile(q_ms, 95)),
            "query_tflops": q_tf, "query_frac_of_bf16_burst": q_tf / peaks["bf16_tflops"],
            "commit_us": 1e6 * c_s, "commit_p95_us": 1e3 * float(np.percentile(c_ms, 95)),
            "commit_hbm_gbs": c_gbs, "commit_frac_of_hbm": c_gbs / peaks["hbm_gbs"],
            "commit_tflops": commit_flops(b, t, h, d) / c_s / 1e12}


def _device_frames(dev, b, t, h, d, n_frames, seed):
    """Seeded synthetic frames generated on the device (timing-only shapes): per frame the 5
    passes' (q, k, v, o) and the gates, with the distributions of the 480p workload."""
    import torch
    g = torch.Generator(device=dev)
    g.manual_seed(seed)
    frames = []
    for _ in range(n_frames):
        passes = []
        for _ in range(QUERIES + 1):
            q, k, v = (torch.randn((b, t, h, d), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
                       for _ in range(3))
            passes.append((q, k, v, torch.empty_like(q)))
        a = torch.sigmoid(2.0 + 0.5 * torch.randn((b, h, t), generator=g, device=dev))
        be = torch.sigmoid(torch.randn((b, h, t), generator=g, device=dev))
        frames.append((passes, a, be))
    wq, wk, wv = ((torch.randn((h, d, d), generator=g, device=dev) / d ** 0.5).to(torch.bfloat16) for _ in range(3))
    return frames, (wq, wk, wv)


def sweep(dev, stream, barrier, peaks, n_frames=30, n_split=30):
    """The token/batch sweep: B in {1, 4} x T in {390, 1560, 3600}, H=12, d=128."""
    import torch

    from softmax_attention_ar_b200.arl2 import ARL2Layer
    rows = []
    for b in (1, 4):
        for t in (390, 1560, 3600):
            act = b * t * H * D * 2
            cycle = max(2, min(8, int(np.ceil(3 * 128e6 / (5 * 3 * act)))))   # > L2 per cycle
            frames, maps = _device_frames(dev, b, t, H, D, cycle, seed=1000 + 10 * b + t)
            layer = ARL2Layer(H, t, D, b)
            layer.set_feature_maps(*maps)

            def frame(i):
                passes, a, be = frames[i % cycle]
                for p in range(QUERIES):
                    layer.query(*passes[p][:3], out=passes[p][3])
                _, k, v, _ = passes[QUERIES]
                layer.commit(k, v, a, be)

            layer.set_launch_overlap(True)
            for i in range(3):
                frame(i)
            fps = _time_windows(frame, stream, 3, n_frames // 3, 3, barrier)
            q_ms, c_ms = _split_times(layer, frames, stream, n_split, barrier)
            st = layer.status()
            ms_frame = 1e3 / statistics.median(fps)   # one frame of all B streams
            row = {"B": b, "T": t, "frames_per_s": b * statistics.median(fps), "ms_per_frame": ms_frame,
                   "frame_frac_of_bf16_burst": (QUERIES * query_flops(b, t, H, D) + commit_flops(b, t, H, D))
                   / (ms_frame / 1e3) / 1e12 / peaks["bf16_tflops"],
                   "status": st, "input_cycle_frames": cycle}
            row.update(_rooflines(q_ms, c_ms, b, t, H, D, peaks))
            rows.append(row)
            layer.close()
            del frames
            torch.cuda.empty_cache()
    return {"what": "4 queries + 1 commit per frame, overlapped; per-kernel times with each launch alone; "
                    "frames/s counts B streams' frames", "H": H, "d": D, "rows": rows}


def stream_leg(layer, frames, stream, barrier, n=240):
    """Per-frame time over n frames (each frame bracketed by events, overlap on inside it) and
    device memory before and after: the layer's cost must not grow with the frame count."""
    import torch
    layer.reset()
    layer.set_launch_overlap(True)
    barrier()
    free0, _ = torch.cuda.mem_get_info()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n)]
    queue_ahead(n * (QUERIES + 3))
    for i, (s, e) in enumerate(ev):
        passes, a, b = frames[i % len(frames)]
        s.record(stream)
        for p in range(QUERIES):
            layer.query(*passes[p][:3], out=passes[p][3])
        _, k, v, _ = passes[QUERIES]
        layer.commit(k, v, a, b)
        e.record(stream)
    barrier()
    free1, _ = torch.cuda.mem_get_info()
    f_us = np.array([1e3 * s.elapsed_time(e) for s, e in ev])
    edge = 50
    return {"frames": n, "us_per_frame_first50": float(f_us[:edge].mean()),
            "us_per_frame_last50": float(f_us[-edge:].mean()),
            "us_per_frame_median": float(np.median(f_us)),
            "slope_us_per_frame": float(np.polyfit(np.arange(n), f_us, 1)[0]),
            "device_free_bytes_before": int(free0), "device_free_bytes_after": int(free1),
            "layer_bytes": layer.memory_bytes, "frame_index_after": layer.frame_index}


def clean_pass_leg(frames, maps, stream, barrier, n_windows=20, window=10, splits=(0,)):
    """The fused clean pass against the two calls it replaces, with launch overlap on:
    frames of 4 denoising queries + the fused clean pass (5 launches) against frames of
    4 queries + the clean pass's query + the commit (6 launches), in alternating windows of
    `window` frames (events around each window); and the clean pass alone, back to back,
    against a query and a commit back to back. Both schedules produce the same outputs:
    the clean pass's o, and S_N."""
    from softmax_attention_ar_b200.arl2 import ARL2Layer
    out = {"what": "per frame: 4 queries + fused clean pass, against 4 queries + query + commit",
           "frames_per_window": window, "windows": n_windows, "splits": []}
    for split in splits:
        fused, sep = ARL2Layer(H, T, D, B), ARL2Layer(H, T, D, B)
        for lay in (fused, sep):
            lay.set_feature_maps(*maps)
            lay.set_launch_overlap(True)
        if split:
            fused.set_clean_split(split)

        def frame_fused(i):
            passes, a, b = frames[i % len(frames)]
            for p in range(QUERIES):
                fused.query(*passes[p][:3], out=passes[p][3])
            q, k, v, o = passes[QUERIES]
            fused.clean_pass(q, k, v, a, b, out=o)

        def frame_sep(i):
            passes, a, b = frames[i % len(frames)]
            for p in range(QUERIES):
                sep.query(*passes[p][:3], out=passes[p][3])
            q, k, v, o = passes[QUERIES]
            sep.query(q, k, v, out=o)
            sep.commit(k, v, a, b)

        def clean_only(i):
            passes, a, b = frames[i % len(frames)]
            q, k, v, o = passes[QUERIES]
            fused.clean_pass(q, k, v, a, b, out=o)

        def pair_only(i):
            passes, a, b = frames[i % len(frames)]
            q, k, v, o = passes[QUERIES]
            sep.query(q, k, v, out=o)
            sep.commit(k, v, a, b)

        for i in range(5):
            frame_fused(i)
            frame_sep(i)
        f_rates, s_rates, c_rates, p_rates = [], [], [], []
        for w in range(n_windows):
            f_rates += _time_windows(frame_fused, stream, 1, window, w * window, barrier)
            s_rates += _time_windows(frame_sep, stream, 1, window, w * window, barrier)
            c_rates += _time_windows(clean_only, stream, 1, window, w * window, barrier)
            p_rates += _time_windows(pair_only, stream, 1, window, w * window, barrier)
        st = max(fused.status(), sep.status())
        if st != 0:
            raise RuntimeError(f"device status {st} in the clean-pass leg")
        med = statistics.median
        out["splits"].append({
            "commit_sms": fused.clean_split, "requested": split,
            "frames_per_s_fused": med(f_rates), "frames_per_s_separate": med(s_rates),
            "us_per_frame_fused": 1e6 / med(f_rates), "us_per_frame_separate": 1e6 / med(s_rates),
            "us_clean_pass_fused": 1e6 / med(c_rates), "us_query_plus_commit": 1e6 / med(p_rates)})
        fused.close()
        sep.close()
    return out


def token_level_leg(frames, maps, stream, barrier, n_windows=10, window=5):
    """Token-level access (the ablation): frames of 4 token-level queries + 1 token-level
    commit, and each call alone in back-to-back windows. A token-level query is three launches
    (the intra branch, the projections, the scan), a commit two (the projections, the scan).
    The scan is fp32 on the CUDA cores: its rate is reported against the SMs' fp32 peak."""
    from softmax_attention_ar_b200.arl2 import ARL2Layer
    lay = ARL2Layer(H, T, D, B)
    lay.set_feature_maps(*maps)

    def frame(i):
        passes, a, b = frames[i % len(frames)]
        for p in range(QUERIES):
            lay.query_token(*passes[p][:3], a, b, out=passes[p][3])
        _, k, v, _ = passes[QUERIES]
        lay.commit_token(k, v, a, b)

    def query_only(i):
        passes, a, b = frames[i % len(frames)]
        lay.query_token(*passes[0][:3], a, b, out=passes[0][3])

    def commit_only(i):
        passes, a, b = frames[i % len(frames)]
        _, k, v, _ = passes[QUERIES]
        lay.commit_token(k, v, a, b)

    for i in range(3):
        frame(i)
    f_rates = _time_windows(frame, stream, n_windows, window, 0, barrier)
    q_rates = _time_windows(query_only, stream, n_windows, window, 0, barrier)
    c_rates = _time_windows(commit_only, stream, n_windows, window, 0, barrier)
    if lay.status() != 0:
        raise RuntimeError("device status in the token-level leg")
    lay.close()
    med = statistics.median
    q_us, c_us = 1e6 / med(q_rates), 1e6 / med(c_rates)
    # Scan arithmetic per token and column of S: k'.s and q'.s (2d flops each) and the update
    # s = alpha s + (beta u) k' (3d flops); a commit has no q'.s.
    scan_q = B * H * T * 7 * D * D
    scan_c = B * H * T * 5 * D * D
    return {"what": "token-level access: per frame 4 queries (intra + projections + scan) and 1 commit "
                    "(projections + scan)",
            "frames_per_s": med(f_rates), "us_per_frame": 1e6 / med(f_rates),
            "us_query": q_us, "us_commit": c_us,
            "scan_flops_query": scan_q, "scan_flops_commit": scan_c,
            "fp32_peak_tflops": FP32_PEAK_TFLOPS,
            "commit_tflops": scan_c / (c_us * 1e-6) / 1e12,
            "commit_frac_of_fp32_peak": scan_c / (c_us * 1e-6) / 1e12 / FP32_PEAK_TFLOPS}


def run_ours(args, rank, world, local_rank):
    import torch
    import torch.distributed as dist

    from softmax_attention_ar_b200.arl2 import ARL2Layer

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    frames, maps, host_frames = make_inputs(dev)
    layer = ARL2Layer(H, T, D, B)
    layer.set_feature_maps(*maps)
    o = torch.empty((B, T, H, D), dtype=torch.bfloat16, device=dev)
    frames = [([p + (o,) for p in passes], a, b) for passes, a, b in frames]
    stream = torch.cuda.current_stream()

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    def step(i):
        passes, a, b = frames[i % CYCLE]
        for p in range(QUERIES):
            layer.query(*passes[p][:3], out=o)
        _, k, v, _ = passes[QUERIES]
        layer.commit(k, v, a, b)

    # Device-resident run. Throughput: the frames back to back, queries and commits
    # overlapping the kernel before them (programmatic dependent launch), only start/end
    # events around exactly `steps` frames.
    layer.set_launch_overlap(True)
    for i in range(args.warmup):
        step(i)
    clocks = ClockSampler(local_rank)
    barrier()
    with clocks:
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        queue_ahead(args.steps * (QUERIES + 1) + 2)
        start.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        end.record(stream)
        barrier()
        # The same window, repeated (the clock sampler keeps running): median and spread.
        reps = _time_windows(step, stream, 20, args.steps, args.warmup + args.steps, barrier)
    elapsed_ms = start.elapsed_time(end)
    # Per-kernel split for the roofline: every launch bracketed by events and run alone.
    split_frames = 200
    q_ms, c_ms = _split_times(layer, frames, stream, split_frames, barrier)
    status = layer.status()
    if status != 0:
        raise RuntimeError(f"device status {status} after the timed region")
    peaks = _peaks()
    stream_info = stream_leg(layer, frames, stream, barrier)
    if layer.status() != 0:
        raise RuntimeError("device status after the streaming leg")
    sweep_info = None if args.no_sweep else sweep(dev, stream, barrier, peaks)

    # End-to-end through the host-buffer entry points (pinned host memory).
    pinned = [([tuple(t.pin_memory() for t in p) for p in passes], a.pin_memory(), b.pin_memory())
              for passes, a, b in host_frames]
    o_host = torch.empty((B, T, H, D), dtype=torch.bfloat16).pin_memory()
    layer.reset()

    def host_step(i):
        passes, a, b = pinned[i % CYCLE]
        for p in range(QUERIES):
            layer.query_host(*passes[p], o_host)
        _, k, v = passes[QUERIES]
        layer.commit_host(k, v, a, b)

    e2e_steps = max(1, min(args.steps, 200)) if not args.no_e2e else 0
    e2e_ms = float("nan")
    if e2e_steps:
        for i in range(min(args.warmup, 3)):
            host_step(i)
        barrier()
        s2, e2 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s2.record(stream)
        for i in range(e2e_steps):
            host_step(i)
        e2.record(stream)
        barrier()
        e2e_ms = s2.elapsed_time(e2)
    act = B * T * H * D * 2
    h2d = (QUERIES * 3 + 2) * act + 2 * B * H * T * 4
    d2h = QUERIES * act

    # Max over ranks.
    elapsed_ms, e2e_ms = max_over_ranks([elapsed_ms, e2e_ms], dev, world)
    if rank != 0:
        return
    value = job_rate(world, B * args.steps, elapsed_ms)
    e2e_value = job_rate(world, B * e2e_steps, e2e_ms) if e2e_steps else None
    k = _rooflines(q_ms, c_ms, B, T, H, D, peaks)
    q_tflops, c_gbs = k["query_tflops"], k["commit_hbm_gbs"]
    frame_s = elapsed_ms / args.steps / 1e3
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": CONFIG,
        "roofline": {"bound": "tensor", "achieved": q_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                     "frac": q_tflops / peaks["bf16_tflops"],
                     "traffic": _profile_traffic("arl2_query_kernel_480p.md", "arl2_query.cu"),
                     "traffic_unit": "DRAM bytes per launch",
                     "kernel": "arl2_query_kernel (one query pass; average over back-to-back query launches)",
                     "algorithmic_flops_per_launch": QUERY_FLOPS,
                     "peak_source": f"bf16_tflops, burst ({peaks['source']})",
                     "frac_of_sustained_peak": q_tflops / peaks["bf16_tflops_sustained"],
                     "frac_of_datasheet_dense_bf16": q_tflops / DATASHEET_BF16_TFLOPS},
        "roofline_commit": {"bound": "hbm", "achieved": c_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                            "frac": c_gbs / peaks["hbm_gbs"],
                            "traffic": _profile_traffic("arl2_commit_kernel_480p.md", "arl2_commit.cu"),
                            "kernel": "arl2_commit_kernel (one commit; average over back-to-back commit launches)",
                            "algorithmic_bytes_per_launch": COMMIT_BYTES,
                            "peak_source": f"hbm_gbs ({peaks['source']})",
                            "tflops": k["commit_tflops"]},
        "frame_roofline": {"what": "4 queries + 1 commit back to back (ms_per_step)",
                           "tflops": FRAME_FLOPS / frame_s / 1e12,
                           "frac_of_bf16_burst": FRAME_FLOPS / frame_s / 1e12 / peaks["bf16_tflops"],
                           "gbs": FRAME_BYTES / frame_s / 1e9,
                           "frac_of_hbm": FRAME_BYTES / frame_s / 1e9 / peaks["hbm_gbs"]},
        "kernels": dict(k, timed_frames=split_frames, launch_overlap="off in this split, on for value", method="windows of 10 frames: 40 queries back to back, then 10 commits back to back, one event pair each"),
        "repeats": {"windows": len(reps), "frames_per_window": args.steps,
                    "median": statistics.median(reps), "min": min(reps), "max": max(reps)},
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps},
        "gpu_launches": args.steps * (QUERIES + 1),   # per frame: the query launches and one commit
        "launch_overlap": "queries and commits launched as programmatic dependents of the kernel before them",
        "clocks": clocks.summary(),
        "stream": stream_info,
    }
    if sweep_info is not None:
        line["sweep"] = sweep_info
    if not args.no_kv_baseline:
        line["kv_cache_baseline"] = kv_cache_baseline(frames, dev, elapsed_ms / args.steps, layer.memory_bytes)
    if not args.no_hybrid_stack:
        line["hybrid_stack"] = hybrid_stack(frames, dev, stream)
    if not args.no_token_level:
        line["token_level"] = token_level_leg(frames, maps, stream, barrier)
    if not args.no_clean_pass:
        line["clean_pass"] = clean_pass_leg(frames, maps, stream, barrier,
                                            splits=tuple(int(x) for x in args.clean_splits.split(",")))
    if world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline()
    print(json.dumps(line), flush=True)
    layer.close()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle CPU baseline")
    ap.add_argument("--no-e2e", action="store_true", help="skip the host-buffer (e2e) measurement")
    ap.add_argument("--no-kv-baseline", action="store_true", help="skip the growing-KV-cache comparison")
    ap.add_argument("--no-sweep", action="store_true", help="skip the token/batch sweep")
    ap.add_argument("--no-hybrid-stack", action="store_true", help="skip the 30-layer hybrid stack timing")
    ap.add_argument("--no-clean-pass", action="store_true", help="skip the fused clean pass comparison")
    ap.add_argument("--no-token-level", action="store_true", help="skip the token-level access timing")
    ap.add_argument("--clean-splits", default="0", help="commit SMs of the fused clean pass to time (0: automatic)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be at least 3")
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_ours(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
