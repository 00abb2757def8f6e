"""Throughput of the Sparse Query Attention core on B200.

One step = one forward pass of the SQA attention core over the encoder-style
long-sequence workload: B=1, N=32768 tokens, d_head=128, non-causal, SQA head
counts H_q=8 query heads sharing H_kv=4 key/value heads (of H=16 head slots),
bf16 Q/K/V ~ N(0,1), fp32 output [B, N, H_q*d_head], through sqa_attn_fwd.
The same kernel at H_q=H=16 (MHA) and the other head-count variants are timed
beside it to give the speed-up that the query-head reduction buys.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl sqa|reference]

Prints ONE JSON line on rank 0.  Multi-GPU runs (torchrun, one rank per GPU)
give every rank its own independent problem of the same size (weak scaling,
no data-path collective); time is the max over ranks.
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
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = {"workload": "sqa_encoder_fwd_32k", "B": 1, "N": 32768, "H_q": 8, "H_kv": 4, "H": 16,
            "d_head": 128, "causal": False, "out": "fp32"}
VARIANTS = {"MHA": (16, 16), "GQA": (16, 4), "SQA": (8, 4), "sSQA": (8, 8), "xSQA": (4, 4)}
METRIC = "SQA attention TFLOP/s and tokens/s at 32k-200k tokens; % of B200 BF16 peak"
L2_FLUSH_BYTES = 256 << 20


def attn_fwd_flops(B, N, H_q, d, causal):
    """Algorithmic FLOPs of the core forward: two contractions of
    2 * B * H_q * P_c * d each, P_c the unmasked (query, key) pairs."""
    P_c = N * (N + 1) // 2 if causal else N * N
    return 4 * B * H_q * P_c * d


def rank_barrier(world):
    """Barrier across the ranks of the default process group (no-op alone)."""
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_max(value, world, device):
    """Max of a float over all ranks (the job's time is its slowest rank's)."""
    if world == 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(world, units_per_rank_step, steps, max_ms):
    """Whole-job rate: every rank processes its own problem each step, the job
    takes as long as the slowest rank (max_ms over `steps` steps)."""
    return world * units_per_rank_step * steps / (max_ms / 1e3)


def device_times(torch, stream, fns, reps, before=None):
    """Device time of each call in `fns`, per repetition: CUDA events on the
    launching stream around every call.  All repetitions are enqueued ahead
    and the host synchronises once at the end, so the host-side launch path
    overlaps the device work of earlier repetitions instead of landing inside
    a timed interval (a per-repetition synchronise leaves the device idle
    while the host launches).  `before` (an L2 flush) runs ahead of each
    repetition, outside its intervals.  Returns one list of ms per call."""
    marks = []
    for _ in range(reps):
        if before is not None:
            before()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(len(fns) + 1)]
        ev[0].record(stream)
        for k, fn in enumerate(fns):
            fn()
            ev[k + 1].record(stream)
        marks.append(ev)
    marks[-1][-1].synchronize()
    return [[ev[k].elapsed_time(ev[k + 1]) for ev in marks] for k in range(len(fns))]


# Nominal dense bf16 tensor peak of a B200 (NVIDIA's sparse figure halved).
NOMINAL_BF16_TFLOPS = 2250.0


def load_peaks():
    """The roofline denominator: the measured cuBLAS bf16 burst rate of this
    pool's B200s (MEASURED_PEAKS.json), else the earlier measurement on the
    pool that stands in for it (1590 TFLOP/s)."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return p.get("bf16_tflops", 1590.0), "measured"
    return 1590.0, "fallback"


# The forward kernel's own sources: its body and the PTX wrappers it inlines.
FWD_KERNEL_SOURCES = ("sqa_fwd_kernel.cuh", "sqa_ptx.cuh")


def csrc_hash(names=FWD_KERNEL_SOURCES):
    """Hash of the forward kernel's sources; the DRAM traffic recorded by ncu
    stays valid only while it is unchanged."""
    h = hashlib.sha256()
    d = os.path.join(ROOT, "sparse_query_attention_b200", "csrc")
    for name in sorted(names):
        with open(os.path.join(d, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def load_traffic():
    """DRAM bytes per launch of the forward kernel from the committed ncu
    summary, valid only while the kernel sources are unchanged."""
    path = os.path.join(ROOT, "profiles", "sqa_fwd_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        t = json.load(f)
    if t.get("csrc_sha") != csrc_hash() or t.get("workload") != WORKLOAD["workload"]:
        return None
    return t.get("dram_bytes_per_launch")


class ClockSampler:
    """SM clock and clock-event reasons sampled while the timed region runs:
    an NVML query every 5 ms from a background thread (a short timed region
    still gets tens of samples); nvidia-smi every 100 ms where NVML is not
    available.  Only reads the GPU's state."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40), ("sw_thermal_slowdown", 0x20),
               ("sw_power_cap", 0x4), ("hw_power_brake_slowdown", 0x80))
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index, period_s=0.005):
        self.gpu = gpu_index
        self.period = period_s
        self.samples = []  # (sm_mhz, reason bitmask)
        self.sm_max = None
        self.proc = None
        self.thread = None
        self.source = None

    def _nvml_loop(self, nv, handle):
        import time as _t
        while not self._stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                except AttributeError:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(handle)
                self.samples.append((float(sm), int(rs)))
            except Exception:  # noqa: BLE001
                pass
            _t.sleep(self.period)

    def __enter__(self):
        self._stop = False
        try:
            import threading

            import pynvml as nv
            nv.nvmlInit()
            handle = nv.nvmlDeviceGetHandleByIndex(self._physical_index())
            self.sm_max = float(nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM))
            self.thread = threading.Thread(target=self._nvml_loop, args=(nv, handle), daemon=True)
            self.thread.start()
            self.source = "nvml every 5 ms"
            return self
        except Exception:  # noqa: BLE001
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self._physical_index()), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.source = "nvidia-smi every 100 ms"
        except OSError:
            self.proc = None
        return self

    def _physical_index(self):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES", "")
        parts = [p.strip() for p in vis.split(",") if p.strip()]
        if parts and parts[0].isdigit() and self.gpu < len(parts):
            return int(parts[self.gpu])
        return self.gpu

    def __exit__(self, *exc):
        self._stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            names = [n for n, _ in self.REASONS[:4]]
            for ln in out.splitlines():
                parts = [p.strip() for p in ln.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm = float(parts[1])
                    self.sm_max = float(parts[2])
                except ValueError:
                    continue
                mask = 0
                for (n, bit), val in zip(self.REASONS[:4], parts[5:9]):
                    if val.lower() == "active":
                        mask |= bit
                self.samples.append((sm, mask))
            del names
        return False

    def summary(self):
        sm = [s for s, _ in self.samples]
        reasons = sorted({n for _, m in self.samples for n, bit in self.REASONS if m & bit})
        counts = {n: sum(1 for _, m in self.samples if m & bit) for n, bit in self.REASONS}
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": self.sm_max,
                "reasons": reasons, "samples": len(sm), "source": self.source,
                "reason_samples": {k: v for k, v in counts.items() if v}}


# ----------------------------------------------------------------------------
# CPU baseline: the oracle as it stands, on a bounded sample of the workload.
# ----------------------------------------------------------------------------
def cpu_baseline(rows_per_head=6144, seed=2):
    import numpy as np
    import torch
    from oracle import attention_forward
    from sqa_inputs import attention_inputs, sample_rows

    w = WORKLOAD
    x = attention_inputs(w["B"], w["N"], w["H_q"], w["H_kv"], w["d_head"], seed, device="cpu")
    q, k, v = (t.double().numpy() for t in (x["q"], x["k"], x["v"]))
    rows = sample_rows(w["N"], rows_per_head, seed)
    try:
        from threadpoolctl import threadpool_info
        cores = max((i.get("num_threads", 1) for i in threadpool_info()), default=1)
    except Exception:  # noqa: BLE001
        cores = os.cpu_count() or 1
    t0 = time.perf_counter()
    attention_forward(q, k, v, w["causal"], 1 / math.sqrt(w["d_head"]), rows=rows)
    dt = time.perf_counter() - t0
    flops = 4 * w["B"] * w["H_q"] * len(rows) * w["N"] * w["d_head"]
    del np, torch
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": int(cores), "kind": "oracle",
            "sample": f"{len(rows)} query rows x {w['H_q']} heads of the N={w['N']} workload "
                      f"({flops / 1e9:.1f} GFLOP, {dt:.2f} s, fp64 numpy)",
            "seconds": dt, "tokens_per_s": w["B"] * len(rows) / dt}


def cpu_baseline_configs():
    """The oracle timed on every configuration of the hot path, on this
    host's cores, within about half a minute: the small causal core (B=2,
    N=256, (4,2), d=32) in full; the decoder layer (B=16, N=1024,
    d_model=256, d=16) forward in full for each of its five head-count
    variants, its backward in full for SQA; the training step (B=4, N=8192,
    (8,4), d=64, forward and backward) on one of its 16 independent
    (batch, KV head) problems, extrapolated x16; the N=32768 encoder core on
    64 sampled query rows per variant and the N=131072 / 200000 core (SQA,
    xSQA) on 4 sampled rows, extrapolated linearly to all N rows (rows are
    independent).  The oracle's inputs at N=131072 and 200000 for MHA's 16
    heads would need several GB of fp64 K and V, so that variant is not
    timed there.  Seconds are per configuration (per step for the layer)."""
    import numpy as np
    from oracle import attention_backward, attention_forward, sqa_layer_backward, sqa_layer_forward
    from sqa_inputs import attention_inputs, layer_inputs, sample_rows

    def np64(t):
        return t.double().numpy()

    out = {}
    x = attention_inputs(2, 256, 4, 2, 32, 0, device="cpu")
    q, k, v = (np64(x[n]) for n in ("q", "k", "v"))
    t0 = time.perf_counter()
    attention_forward(q, k, v, True, 1 / math.sqrt(32))
    out["causal_core_b2_n256"] = {"timed": "full", "fwd_seconds": time.perf_counter() - t0}
    c = LAYER
    B, N, dm, dh = c["B"], c["N"], c["d_model"], c["d_head"]
    lay = {}
    for name in ("GQA", "SQA", "sSQA", "xSQA", "xSMQA"):
        hq, hkv = LAYER_VARIANTS[name]
        xl = layer_inputs(B, N, dm, hq, hkv, dh, seed=1, device="cpu")
        a = [np64(xl[k]) for k in ("x", "wq", "wk", "wv", "wo")]
        t0 = time.perf_counter()
        sqa_layer_forward(*a, B, N, hq, hkv, dh, causal=True)
        lay[name] = {"fwd_seconds": time.perf_counter() - t0}
        if name == "SQA":
            dy = np.random.default_rng(11).standard_normal((B * N, dm))
            t0 = time.perf_counter()
            sqa_layer_backward(*a, dy, B, N, hq, hkv, dh, causal=True)
            lay[name]["bwd_seconds"] = time.perf_counter() - t0
    out["decoder_layer_b16_n1024"] = {"timed": "full (backward for SQA only)", "variants": lay}
    t = TRAIN
    G = t["H_q"] // t["H_kv"]
    xt = attention_inputs(1, t["N"], t["H_q"], t["H_kv"], t["d_head"], 4, with_dout=True, device="cpu")
    q, do = (np64(xt[n][:, :, :G]) for n in ("q", "do"))  # KV head 0 and its G query heads
    k, v = (np64(xt[n][:, :, :1]) for n in ("k", "v"))
    sc = 1 / math.sqrt(t["d_head"])
    parts = t["B"] * t["H_kv"]
    t0 = time.perf_counter()
    attention_forward(q, k, v, True, sc)
    t1 = time.perf_counter()
    attention_backward(q, k, v, do, True, sc)
    t2 = time.perf_counter()
    out["training_step_b4_n8192"] = {"timed": f"1 of {parts} (batch, KV head) problems, extrapolated x{parts}",
                                     "fwd_seconds": parts * (t1 - t0), "bwd_seconds": parts * (t2 - t1)}
    del xt, q, k, v, do
    w = WORKLOAD
    enc = {}
    rows = sample_rows(w["N"], 64, 2)
    for name, (hq, hkv) in VARIANTS.items():
        xe = attention_inputs(1, w["N"], hq, hkv, w["d_head"], 2, device="cpu")
        q, k, v = (np64(xe[n]) for n in ("q", "k", "v"))
        del xe
        t0 = time.perf_counter()
        attention_forward(q, k, v, False, 1 / math.sqrt(w["d_head"]), rows=rows)
        dt = time.perf_counter() - t0
        enc[name] = {"fwd_seconds": dt * w["N"] / len(rows), "sample_seconds": dt}
        del q, k, v
    out["encoder_core_n32768"] = {"timed": f"{len(rows)} sampled query rows, extrapolated to N={w['N']}",
                                  "variants": enc}
    lng = {}
    for N in LONG["N"]:
        rows = sample_rows(N, 4, 3)
        per = {}
        for name in ("SQA", "xSQA"):
            hq, hkv = LONG_VARIANTS[name]
            xe = attention_inputs(1, N, hq, hkv, LONG["d_head"], 3, device="cpu")
            q, k, v = (np64(xe[n]) for n in ("q", "k", "v"))
            del xe
            t0 = time.perf_counter()
            attention_forward(q, k, v, False, 1 / math.sqrt(LONG["d_head"]), rows=rows)
            dt = time.perf_counter() - t0
            per[name] = {"fwd_seconds": dt * N / len(rows), "sample_seconds": dt}
            del q, k, v
        lng[str(N)] = per
    out["long_core"] = {"timed": "4 sampled query rows, extrapolated to N (MHA not timed)", "by_N": lng}
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        b = cpu_baseline(rows_per_head=16 if args.steps > 3 else 32)
        if i >= args.warmup:
            per_step.append(b)
        base = b
    secs = sum(b["seconds"] for b in per_step)
    flops = sum(b["value"] * b["seconds"] * 1e12 for b in per_step)
    val = flops / secs / 1e12
    line = {"metric": METRIC, "value": val, "unit": "TFLOP/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * secs / len(per_step),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(WORKLOAD, sample=base["sample"]),
            "cpu_baseline": {"value": val, "unit": "TFLOP/s", "cores": base["cores"], "kind": "oracle",
                             "sample": base["sample"]},
            "e2e": {"value": val, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------
TRAIN = {"B": 4, "N": 8192, "H_q": 8, "H_kv": 4, "d_head": 64, "causal": True}


LONG = {"B": 1, "d_head": 128, "causal": False, "N": (131072, 200000)}
LONG_VARIANTS = {"MHA": (16, 16), "SQA": (8, 4), "xSQA": (4, 4)}


def time_long_sequences(sqa, torch, stream, dev, reps=3):
    """Non-causal core forward at N = 131072 and 200000 (B=1, d=128) for MHA,
    SQA and xSQA on the same kernel: the long-sequence end of the 32k-200k
    range.  Inputs are larger than L2, so no flush is needed."""
    from sqa_inputs import attention_inputs

    c = LONG
    d = c["d_head"]
    res = {}
    for N in c["N"]:
        # The variants are timed round-robin (one launch each per round) so
        # that the speed-up over MHA compares launches at the same clock.
        data, fns = {}, []
        for name, (hq, hkv) in LONG_VARIANTS.items():
            x = attention_inputs(1, N, hq, hkv, d, seed=3, device=dev)
            o = torch.empty((1, N, hq * d), dtype=torch.float32, device=dev)
            data[name] = (x, o)

            def fwd(x=x, o=o, hq=hq, hkv=hkv):
                sqa.sqa_attn_fwd(x["q"], x["k"], x["v"], o, 1, N, hq, hkv, d, False, 1 / math.sqrt(d),
                                 stream=stream)

            fwd()
            fns.append(fwd)
        times = device_times(torch, stream, fns, reps)
        per = {}
        for (name, (hq, hkv)), t in zip(LONG_VARIANTS.items(), times):
            ms = statistics.median(t)
            per[name] = {"H_q": hq, "H_kv": hkv, "ms": ms,
                         "tflops": attn_fwd_flops(1, N, hq, d, False) / ms / 1e9, "tokens_per_s": N / (ms / 1e3)}
        del data, fns
        for name in per:
            per[name]["speedup_vs_mha"] = per["MHA"]["ms"] / per[name]["ms"]
        res[str(N)] = per
    sqa.sqa_device_status(stream)
    return {"config": {"B": 1, "d_head": d, "causal": False}, "by_N": res}


WINDOW = {"B": 1, "N": 131072, "d_head": 128, "windows": {"causal_4096": (4095, 0), "local_2048": (2048, 2048)}}


def window_pairs(N, left, right):
    """Visible (query, key) pairs of a band t - left <= u <= t + right:
    the sum over t of min(N - 1, t + right) - max(0, t - left) + 1."""
    import numpy as np

    t = np.arange(N, dtype=np.int64)
    return int((np.minimum(N - 1, t + right) - np.maximum(0, t - left) + 1).sum())


def time_windowed(sqa, torch, stream, dev, reps=5):
    """Sliding-window SQA at N = 131072 (B=1, d=128): a causal window of 4096
    keys and a symmetric local window of +-2048, forward for MHA, SQA and
    xSQA on the same kernel, and the SQA training step (forward + backward)
    with the causal window.  FLOPs count visible pairs only
    (4 * H_q * P_w * d forward, 8 * H_q * P_w * d backward), so a rate close
    to the dense kernel's means the skipped tiles cost nothing."""
    from sqa_inputs import attention_inputs

    c = WINDOW
    N, d = c["N"], c["d_head"]
    sc = 1 / math.sqrt(d)

    def med(fn):
        fn()
        return statistics.median(device_times(torch, stream, [fn], reps)[0])

    res = {}
    inputs = {name: attention_inputs(1, N, hq, hkv, d, seed=3, device=dev)
              for name, (hq, hkv) in LONG_VARIANTS.items()}
    outs = {name: torch.empty((1, N, hq, d), dtype=torch.float32, device=dev)
            for name, (hq, hkv) in LONG_VARIANTS.items()}
    for wname, (left, right) in c["windows"].items():
        P_w = window_pairs(N, left, right)

        def fwd(name, left=left, right=right):
            hq, hkv = LONG_VARIANTS[name]
            x, o = inputs[name], outs[name]
            return lambda: sqa.sqa_attn_fwd_window(x["q"], x["k"], x["v"], o, sqa.SQA_DT_F32, None, 1, N, hq, hkv,
                                                   d, left, right, sc, stream=stream)

        # Round-robin (one launch of each variant per round), so that every
        # variant sees the same clock at the power cap.
        fns = [fwd(name) for name in LONG_VARIANTS]
        for fn in fns:
            fn()
        times = device_times(torch, stream, fns, reps)
        per = {}
        for name, t in zip(LONG_VARIANTS, times):
            hq, hkv = LONG_VARIANTS[name]
            ms = statistics.median(t)
            per[name] = {"H_q": hq, "H_kv": hkv, "ms": ms, "tflops": 4 * hq * P_w * d / ms / 1e9,
                         "tokens_per_s": N / (ms / 1e3)}
        for name in per:
            per[name]["speedup_vs_mha"] = per["MHA"]["ms"] / per[name]["ms"]
        res[wname] = {"left": left, "right": right, "visible_pairs": P_w, "forward": per}
    del inputs, outs
    # SQA training step with the causal window.
    left, right = c["windows"]["causal_4096"]
    hq, hkv = LONG_VARIANTS["SQA"]
    P_w = window_pairs(N, left, right)
    x = attention_inputs(1, N, hq, hkv, d, seed=3, with_dout=True, device=dev)
    o = torch.empty((1, N, hq, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((1, hq, N), dtype=torch.float32, device=dev)
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.bfloat16, device=dev) for t in (x["q"], x["k"], x["v"]))
    wsb = sqa.sqa_attn_bwd_workspace_size(1, N, hq, hkv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    BF = sqa.SQA_DT_BF16
    fwd_ms = med(lambda: sqa.sqa_attn_fwd_window(x["q"], x["k"], x["v"], o, BF, lse, 1, N, hq, hkv, d, left, right,
                                                 sc, stream=stream))
    bwd_ms = med(lambda: sqa.sqa_attn_bwd_window(x["q"], x["k"], x["v"], o, BF, x["do"], lse, dq, dk, dv, BF, 1, N,
                                                 hq, hkv, d, left, right, sc, ws, wsb, stream=stream))
    res["sqa_train_causal_4096"] = {"fwd_ms": fwd_ms, "bwd_ms": bwd_ms,
                                    "fwd_tflops": 4 * hq * P_w * d / fwd_ms / 1e9,
                                    "bwd_tflops": 8 * hq * P_w * d / bwd_ms / 1e9,
                                    "tokens_per_s": N / ((fwd_ms + bwd_ms) / 1e3)}
    sqa.sqa_device_status(stream)
    return {"config": {"B": 1, "N": N, "d_head": d}, "windows": res}


CROSS = {"B": 1, "N_q": 32768, "N_kv": 8192, "d_head": 128}


def time_cross(sqa, torch, stream, dev, reps=5):
    """Cross / memory attention, N_q = 32768 queries against N_kv = 8192 keys
    of another sequence (B=1, d=128, no mask): forward for MHA, SQA and xSQA
    on the same kernel, and the SQA backward.  FLOPs 4 * H_q * N_q * N_kv * d
    forward, 8 * ... backward."""
    from sqa_inputs import cross_attention_inputs

    c = CROSS
    B, Nq, Nkv, d = c["B"], c["N_q"], c["N_kv"], c["d_head"]
    sc = 1 / math.sqrt(d)

    def med(fn):
        fn()
        return statistics.median(device_times(torch, stream, [fn], reps)[0])

    # Forward of the three variants timed round-robin (one launch of each
    # per round), then the SQA backward.
    res, data, fns = {}, {}, []
    BF = sqa.SQA_DT_BF16
    for name, (hq, hkv) in LONG_VARIANTS.items():
        x = cross_attention_inputs(B, Nq, Nkv, hq, hkv, d, seed=6, with_dout=name == "SQA", device=dev)
        o = torch.empty((B, Nq, hq, d), dtype=torch.bfloat16, device=dev)
        lse = torch.empty((B, hq, Nq), dtype=torch.float32, device=dev)
        data[name] = (x, o, lse)

        def fwd(x=x, o=o, lse=lse, hq=hq, hkv=hkv):
            sqa.sqa_attn_fwd_cross(x["q"], x["k"], x["v"], o, BF, lse, B, Nq, Nkv, hq, hkv, d, sc, stream=stream)

        fwd()
        fns.append(fwd)
    times = device_times(torch, stream, fns, reps)
    for (name, (hq, hkv)), t in zip(LONG_VARIANTS.items(), times):
        ms = statistics.median(t)
        flops = 4 * B * hq * Nq * Nkv * d
        res[name] = {"H_q": hq, "H_kv": hkv, "fwd_ms": ms, "fwd_tflops": flops / ms / 1e9}
    x, o, lse = data["SQA"]
    hq, hkv = LONG_VARIANTS["SQA"]
    dq, dk, dv = (torch.empty(t.shape, dtype=torch.bfloat16, device=dev) for t in (x["q"], x["k"], x["v"]))
    wsb = sqa.sqa_attn_bwd_workspace_size(B, Nq, hq, hkv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    bms = med(lambda: sqa.sqa_attn_bwd_cross(x["q"], x["k"], x["v"], o, BF, x["do"], lse, dq, dk, dv, BF, B, Nq, Nkv,
                                             hq, hkv, d, sc, ws, wsb, stream=stream))
    res["SQA"].update({"bwd_ms": bms, "bwd_tflops": 8 * B * hq * Nq * Nkv * d / bms / 1e9})
    del data, fns
    for name in res:
        res[name]["fwd_speedup_vs_mha"] = res["MHA"]["fwd_ms"] / res[name]["fwd_ms"]
    sqa.sqa_device_status(stream)
    return {"config": dict(c), "variants": res}


DECODE = {"B": 16, "L": 32768, "n_new": 1, "d_head": 128}
DECODE_VARIANTS = {"MHA": (16, 16), "GQA": (16, 4), "SQA": (8, 4), "xSQA": (4, 4), "xSMQA": (4, 1)}


PROJ = {"M": 32768, "N": 4096, "K": 4096}


def proj_operands(torch, dev):
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    c = PROJ
    x = torch.randn((c["M"], c["K"]), generator=g, device=dev).to(torch.bfloat16)
    w = (0.02 * torch.randn((c["N"], c["K"]), generator=g, device=dev)).to(torch.bfloat16)
    return x, w


def time_projection(sqa, torch, stream, dev, reps=10):
    """The projection GEMM (Y = X W^T, bf16 in, bf16 out, fp32 accumulate) at
    M=32768, N=K=4096, against torch.matmul (cuBLAS) on the same operands, as
    context for the measured bf16 peak.  Operands (0.5 GB) exceed the L2."""
    c = PROJ
    M, N, K = c["M"], c["N"], c["K"]
    x, w = proj_operands(torch, dev)
    y = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ours = lambda: sqa.sqa_proj(x, w, None, y, sqa.SQA_DT_BF16, M, K, N, stream=stream)
    ref = lambda: torch.matmul(x, w.t(), out=y)
    for _ in range(3):
        ours()
        ref()
    t_ours, t_ref = device_times(torch, stream, [ours, ref], reps)
    flops = 2.0 * M * N * K
    ms_o, ms_r = statistics.median(t_ours), statistics.median(t_ref)
    sqa.sqa_device_status(stream)
    return {"config": dict(c), "sqa_proj_ms": ms_o, "sqa_proj_tflops": flops / ms_o / 1e9,
            "cublas_ms": ms_r, "cublas_tflops": flops / ms_r / 1e9}


def secondary_leg(fn):
    """Runs one secondary measurement; an exception becomes {"error": ...}
    in the JSON line instead of ending the run."""
    try:
        return fn()
    except Exception as e:  # noqa: BLE001 - any failure is reported, none is hidden
        return {"error": f"{type(e).__name__}: {e}"[:400]}


def load_hbm_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f).get("hbm_gbs", 6650.0), "measured"
    return 6650.0, "fallback"


def time_decode(sqa, torch, stream, dev, reps=10):
    """One decode step (n_new = 1) for B = 16 sequences with 32768 cached
    tokens, d = 128, per head-count variant.  HBM-bound: algorithmic bytes
    are the K and V cache (2 * B * L * H_kv * d bf16) plus Q and O; the cache
    (256 MiB at xSMQA's single KV head, 4 GiB at MHA) is larger than the L2 at
    every variant, so no flush is added.  Steps run back to back, as decode
    steps do in serving.  Reported against the measured copy bandwidth."""
    c = DECODE
    B, L, n_new, d = c["B"], c["L"], c["n_new"], c["d_head"]
    peak, kind = load_hbm_peak()
    res = {}
    for name, (hq, hkv) in DECODE_VARIANTS.items():
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        q = torch.randn((B, n_new, hq, d), generator=g, device=dev).to(torch.bfloat16)
        kc = torch.randn((B, L, hkv, d), generator=g, device=dev).to(torch.bfloat16)
        vc = torch.randn((B, L, hkv, d), generator=g, device=dev).to(torch.bfloat16)
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        out = torch.empty((B, n_new, hq, d), dtype=torch.bfloat16, device=dev)
        wsb = sqa.sqa_attn_decode_workspace_size(B, n_new, hq, hkv, d, L)
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)

        def step():
            sqa.sqa_attn_decode(q, kc, vc, lens, out, sqa.SQA_DT_BF16, None, B, n_new, hq, hkv, d, L,
                                1 / math.sqrt(d), ws if wsb else None, wsb, stream=stream)

        for _ in range(3):
            step()
        ms = statistics.median(device_times(torch, stream, [step], reps)[0])
        nbytes = 2 * B * L * hkv * d * 2 + 2 * B * n_new * hq * d * 2
        res[name] = {"H_q": hq, "H_kv": hkv, "ms": ms, "gbs": nbytes / ms / 1e6, "frac_hbm": nbytes / ms / 1e6 / peak,
                     "tokens_per_s": B * n_new / (ms / 1e3)}
        del q, kc, vc, out, ws
    sqa.sqa_device_status(stream)
    return {"config": dict(c), "hbm_peak_gbs": peak, "hbm_peak_source": f"{kind} copy", "variants": res}


LAYER = {"B": 16, "N": 1024, "d_model": 256, "d_head": 16, "causal": True}
LAYER_VARIANTS = {"MHA": (16, 16), "GQA": (16, 4), "SQA": (8, 4), "sSQA": (8, 8), "xSQA": (4, 4), "xSMQA": (4, 1)}


def decoder_layer_step(sqa, torch, stream, dev, name):
    """The small decoder attention layer (B=16, N=1024, d_model=256,
    d_head=16, causal) at one head-count variant: returns its forward and
    its backward as two closures over their own buffers.  The input
    projection is fused: one GEMM with the concatenated weight [Wq; Wk; Wv]
    writes a packed QKV buffer that the attention reads in place; the
    backward writes packed dQKV, so dX and d[Wq; Wk; Wv] are one GEMM each."""
    from sqa_inputs import layer_inputs

    c = LAYER
    B, N, dm, dh = c["B"], c["N"], c["d_model"], c["d_head"]
    hq, hkv = LAYER_VARIANTS[name]
    M = B * N
    x = layer_inputs(B, N, dm, hq, hkv, dh, seed=1, device=dev)
    W = (hq + 2 * hkv) * dh
    w_qkv = torch.cat([x["wq"], x["wk"], x["wv"]], dim=0).contiguous()
    qkv = torch.empty((M, W), dtype=torch.bfloat16, device=dev)
    o = torch.empty((M, hq * dh), dtype=torch.bfloat16, device=dev)
    y = torch.empty((M, dm), dtype=torch.float32, device=dev)
    lse = torch.empty((B, hq, N), dtype=torch.float32, device=dev)
    gen = torch.Generator(device=dev)
    gen.manual_seed(11)
    dy = torch.randn((M, dm), generator=gen, device=dev).to(torch.bfloat16)
    do = torch.empty_like(o)
    dqkv = torch.empty_like(qkv)
    dx = torch.empty((M, dm), dtype=torch.float32, device=dev)
    dw_qkv = torch.empty((W, dm), dtype=torch.float32, device=dev)
    dwo = torch.empty((dm, hq * dh), dtype=torch.float32, device=dev)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, hq, hkv, dh)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
    KC, MN, BF, F32 = sqa.SQA_K_CONTIGUOUS, sqa.SQA_MN_CONTIGUOUS, sqa.SQA_DT_BF16, sqa.SQA_DT_F32
    sc = 1 / math.sqrt(dh)

    def layer():
        sqa.sqa_proj(x["x"], w_qkv, None, qkv, BF, M, dm, W, stream=stream)
        sqa.sqa_attn_fwd_packed(qkv, o, BF, lse, B, N, hq, hkv, dh, True, sc, stream=stream)
        sqa.sqa_proj(o, x["wo"], None, y, F32, M, hq * dh, dm, stream=stream)

    def layer_backward():
        sqa.sqa_gemm(dy, KC, x["wo"], MN, None, do, BF, False, M, hq * dh, dm, stream=stream)
        sqa.sqa_gemm(dy, MN, o, MN, None, dwo, F32, False, dm, hq * dh, M, stream=stream)
        sqa.sqa_attn_bwd_packed(qkv, o, BF, do, lse, dqkv, BF, B, N, hq, hkv, dh, True, sc, ws, wsb,
                                stream=stream)
        sqa.sqa_gemm(dqkv, KC, w_qkv, MN, None, dx, F32, False, M, dm, W, stream=stream)
        sqa.sqa_gemm(dqkv, MN, x["x"], MN, None, dw_qkv, F32, False, W, dm, M, stream=stream)

    return layer, layer_backward


def time_decoder_layer(sqa, torch, stream, flush, dev, reps=5):
    """Forward and training step of the small decoder attention layer (B=16,
    N=1024, d_model=256, d_head=16, causal; decoder_layer_step), per
    head-count variant (median of reps, L2 flushed).  Forward 3 launches,
    training step 10."""
    c = LAYER
    B, N, dm, dh = c["B"], c["N"], c["d_model"], c["d_head"]
    M = B * N
    P_c = N * (N + 1) // 2
    out = {}
    for name, (hq, hkv) in LAYER_VARIANTS.items():
        layer, layer_backward = decoder_layer_step(sqa, torch, stream, dev, name)

        def timed(fn):
            for _ in range(3):
                fn()
            return statistics.median(device_times(torch, stream, [fn], reps, before=lambda: flush.fill_(3))[0])

        def step():
            layer()
            layer_backward()

        ms = timed(layer)
        ms_train = timed(step)
        proj_f = 2 * M * dm * (hq + 2 * hkv) * dh + 2 * M * hq * dh * dm
        attn_f = 4 * B * hq * P_c * dh
        flops = proj_f + attn_f
        train_flops = 3 * proj_f + 3 * attn_f  # backward: 2x projections, 2x core (algorithmic)
        out[name] = {"H_q": hq, "H_kv": hkv, "ms": ms, "tflops": flops / ms / 1e9, "tokens_per_s": M / (ms / 1e3),
                     "train_ms": ms_train, "train_tflops": train_flops / ms_train / 1e9,
                     "train_tokens_per_s": M / (ms_train / 1e3)}
    for name in out:
        out[name]["speedup_vs_gqa"] = out["GQA"]["ms"] / out[name]["ms"]
        out[name]["train_speedup_vs_gqa"] = out["GQA"]["train_ms"] / out[name]["train_ms"]
    sqa.sqa_device_status(stream)
    return {"config": dict(c), "launches_forward": 3, "launches_training_step": 10, "fused_qkv": True, "variants": out}


def time_training_step(sqa, torch, stream, flush, dev, reps=5):
    """Causal SQA core forward + backward at B=4, N=8192, H_q=8, H_kv=4, d=64
    (bf16 inputs, fp32 gradients): median over reps, L2 flushed before each."""
    from sqa_inputs import attention_inputs

    t = TRAIN
    B, N, H_q, H_kv, d = t["B"], t["N"], t["H_q"], t["H_kv"], t["d_head"]
    scale = 1 / math.sqrt(d)
    x = attention_inputs(B, N, H_q, H_kv, d, seed=4, with_dout=True, device=dev)
    o = torch.empty((B, N, H_q, d), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((B, H_q, N), dtype=torch.float32, device=dev)
    dq = torch.empty((B, N, H_q, d), dtype=torch.float32, device=dev)
    dk = torch.empty((B, N, H_kv, d), dtype=torch.float32, device=dev)
    dv = torch.empty_like(dk)
    wsb = sqa.sqa_attn_bwd_workspace_size(B, N, H_q, H_kv, d)
    ws = torch.empty(wsb, dtype=torch.uint8, device=dev)

    def fwd():
        sqa.sqa_attn_fwd_ex(x["q"], x["k"], x["v"], o, sqa.SQA_DT_BF16, lse, B, N, H_q, H_kv, d, True, scale,
                            stream=stream)

    def bwd():
        sqa.sqa_attn_bwd(x["q"], x["k"], x["v"], o, sqa.SQA_DT_BF16, x["do"], lse, dq, dk, dv, sqa.SQA_DT_F32,
                         B, N, H_q, H_kv, d, True, scale, ws, wsb, stream=stream)

    for _ in range(3):
        fwd()
        bwd()
    tf, tb = device_times(torch, stream, [fwd, bwd], reps, before=lambda: flush.fill_(2))
    sqa.sqa_device_status(stream)
    ms_f, ms_b = statistics.median(tf), statistics.median(tb)
    f_fwd = attn_fwd_flops(B, N, H_q, d, True)
    f_bwd = 2 * f_fwd  # dP, dV, dQ, dK; recomputation of S not credited
    return {"config": dict(t), "fwd_ms": ms_f, "bwd_ms": ms_b, "fwd_tflops": f_fwd / ms_f / 1e9,
            "bwd_tflops": f_bwd / ms_b / 1e9, "bwd_tflops_fa_convention": 2.5 * f_fwd / ms_b / 1e9,
            "step_tflops": (f_fwd + f_bwd) / (ms_f + ms_b) / 1e9,
            "tokens_per_s": B * N / ((ms_f + ms_b) / 1e3)}
def run_sqa(args):
    import torch
    import torch.distributed as dist

    import sparse_query_attention_b200 as sqa
    from sqa_inputs import attention_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    dev = torch.device("cuda", local)
    stream = torch.cuda.current_stream(dev)
    w = WORKLOAD
    B, N, H_q, H_kv, d = w["B"], w["N"], w["H_q"], w["H_kv"], w["d_head"]
    scale = 1 / math.sqrt(d)
    flops_step = attn_fwd_flops(B, N, H_q, d, w["causal"])

    x = attention_inputs(B, N, H_q, H_kv, d, seed=2 + rank, device=dev)
    out = torch.empty((B, N, H_q * d), dtype=torch.float32, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)

    def step(q, k, v, o, h_q=H_q, h_kv=H_kv):
        sqa.sqa_attn_fwd(q, k, v, o, B, N, h_q, h_kv, d, w["causal"], scale, stream=stream)

    def barrier():
        rank_barrier(world)
        torch.cuda.synchronize(dev)

    def max_over_ranks(val):
        return dist_max(val, world, dev)

    for _ in range(args.warmup):
        step(x["q"], x["k"], x["v"], out)
    sqa.sqa_device_status(stream)

    # --- timed region: K steps, L2 flushed between steps (not timed) -------
    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    barrier()
    with ClockSampler(local) as clocks:
        for i in range(args.steps):
            flush.fill_(i & 0xFF)
            starts[i].record(stream)
            step(x["q"], x["k"], x["v"], out)
            ends[i].record(stream)
        barrier()
    sqa.sqa_device_status(stream)
    per_launch_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(per_launch_ms))
    ms_per_step = total_ms / args.steps
    value = weak_scaling_rate(world, flops_step, args.steps, total_ms) / 1e12
    tokens_per_s = weak_scaling_rate(world, B * N, args.steps, total_ms)

    # --- end to end through the C ABI with host buffers --------------------
    # Every step copies its inputs from pinned host memory and reads its
    # output back.  Measured two ways: serial (copy in, compute, copy out,
    # one stream) and pipelined (two device buffer sets; host-to-device
    # copies of step i+1 and the read-back of step i-1 on their own streams
    # overlap step i's kernel).  The pipelined number is the headline.
    hq, hk, hv = (t.cpu().pin_memory() for t in (x["q"], x["k"], x["v"]))
    ho = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    dsets = [tuple(torch.empty_like(t) for t in (x["q"], x["k"], x["v"])) for _ in range(2)]
    douts = [torch.empty_like(out) for _ in range(2)]
    # A fixed 50-step window (reported as e2e.steps), whatever --steps is:
    # the pipeline's first copy-in and last read-back are not overlapped, and
    # over 50 steps they cost ~3 % instead of ~7 % at 20.
    e2e_steps = 50

    def serial_step():
        dq_, dk_, dv_ = dsets[0]
        for hsrc, ddst in ((hq, dq_), (hk, dk_), (hv, dv_)):
            ddst.copy_(hsrc, non_blocking=True)
        step(dq_, dk_, dv_, douts[0])
        ho[0].copy_(douts[0], non_blocking=True)

    for _ in range(2):
        serial_step()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        serial_step()
    e1.record(stream)
    barrier()
    e2e_serial_ms = max_over_ranks(e0.elapsed_time(e1))

    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)

    def pipelined(n):
        h2d_done = [torch.cuda.Event() for _ in range(2)]
        comp_done = [torch.cuda.Event() for _ in range(2)]
        d2h_done = [torch.cuda.Event() for _ in range(2)]
        used = [False, False]
        s_in.wait_stream(stream)  # nothing starts before the timing event on the compute stream
        for i in range(n):
            sl = i % 2
            dq_, dk_, dv_ = dsets[sl]
            with torch.cuda.stream(s_in):
                if used[sl]:
                    s_in.wait_event(comp_done[sl])  # the kernel that read this buffer set is done
                for hsrc, ddst in ((hq, dq_), (hk, dk_), (hv, dv_)):
                    ddst.copy_(hsrc, non_blocking=True)
                h2d_done[sl].record(s_in)
            stream.wait_event(h2d_done[sl])
            if used[sl]:
                stream.wait_event(d2h_done[sl])  # this output buffer has been read back
            step(dq_, dk_, dv_, douts[sl])
            comp_done[sl].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(comp_done[sl])
                ho[sl].copy_(douts[sl], non_blocking=True)
                d2h_done[sl].record(s_out)
            used[sl] = True
        stream.wait_stream(s_in)
        stream.wait_stream(s_out)

    pipelined(2)
    barrier()
    e0.record(stream)
    pipelined(e2e_steps)
    e1.record(stream)
    barrier()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1))
    e2e_value = weak_scaling_rate(world, flops_step, e2e_steps, e2e_ms) / 1e12
    e2e_serial = weak_scaling_rate(world, flops_step, e2e_steps, e2e_serial_ms) / 1e12
    h2d = sum(t.numel() * t.element_size() for t in (hq, hk, hv))
    d2h = ho[0].numel() * ho[0].element_size()

    # --- head-count variants on the same kernel (speed-up vs H_q = H) ------
    # Timed round-robin, one launch of every variant per round (L2 flushed
    # before each): on a GPU at its power cap the clock drifts over tens of
    # milliseconds, and variants timed one block after another would compare
    # different clocks.
    vin = {}
    for name, (vq, vkv) in VARIANTS.items():
        xv = attention_inputs(B, N, vq, vkv, d, seed=2, device=dev)
        vin[name] = (xv, torch.empty((B, N, vq * d), dtype=torch.float32, device=dev))
        for _ in range(2):
            step(xv["q"], xv["k"], xv["v"], vin[name][1], vq, vkv)
    names = list(VARIANTS)

    def launcher(nm):
        vq, vkv = VARIANTS[nm]
        xv, ov = vin[nm]
        return lambda: step(xv["q"], xv["k"], xv["v"], ov, vq, vkv)

    fns = []
    for nm in names:  # a flush, then the launch: one timed interval per variant per round
        fns += [lambda: flush.fill_(1), launcher(nm)]
    rounds = device_times(torch, stream, fns, 7)
    variants = {}
    for i, nm in enumerate(names):
        vq, vkv = VARIANTS[nm]
        ms = statistics.median(rounds[2 * i + 1])
        variants[nm] = {"H_q": vq, "H_kv": vkv, "ms": ms,
                        "tflops": attn_fwd_flops(B, N, vq, d, w["causal"]) / (ms / 1e3) / 1e12}
    del vin
    for name in variants:
        variants[name]["speedup_vs_mha"] = variants["MHA"]["ms"] / variants[name]["ms"]
        variants[name]["ideal_speedup"] = VARIANTS["MHA"][0] / variants[name]["H_q"]
    sqa.sqa_device_status(stream)
    # The secondary legs (no collectives): a failure in one is recorded in
    # its place in the line instead of ending the run, so the measurement
    # above is still reported.
    training = secondary_leg(lambda: time_training_step(sqa, torch, stream, flush, dev))
    layer = secondary_leg(lambda: time_decoder_layer(sqa, torch, stream, flush, dev))
    long_seq = secondary_leg(lambda: time_long_sequences(sqa, torch, stream, dev))
    windowed = secondary_leg(lambda: time_windowed(sqa, torch, stream, dev))
    decode = secondary_leg(lambda: time_decode(sqa, torch, stream, dev))
    cross = secondary_leg(lambda: time_cross(sqa, torch, stream, dev))
    projection = secondary_leg(lambda: time_projection(sqa, torch, stream, dev))

    peak, peak_kind = load_peaks()
    achieved = flops_step / (statistics.mean(per_launch_ms) / 1e3) / 1e12
    traffic = load_traffic()
    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(WORKLOAD, parallelism=f"independent problems x{world}",
                       l2="flushed between timed steps (256 MiB write)"),
        "tokens_per_s": tokens_per_s,
        "pct_of_bf16_peak": 100 * achieved / peak,
        "pct_of_nominal_bf16_peak": 100 * achieved / NOMINAL_BF16_TFLOPS,
        "roofline": {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                     "frac": achieved / peak, "traffic": traffic, "peak_source": f"{peak_kind} bf16 burst"},
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "steps": e2e_steps, "mode": "pipelined: copies of neighbouring steps overlap the kernel",
                "ms_per_step": e2e_ms / e2e_steps, "kernel_ms_per_step": ms_per_step,
                "serial_value": e2e_serial},
        "gpu_launches": args.steps,
        "variants": variants,
        "training_step": training,
        "decoder_layer": layer,
        "long_sequences": long_seq,
        "windowed": windowed,
        "decode": decode,
        "cross": cross,
        "projection": projection,
        "clocks": clocks.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = {k: v for k, v in cpu_baseline().items() if k not in ("seconds",)}
        line["cpu_baseline"]["configs"] = secondary_leg(cpu_baseline_configs)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_profile(args):
    """Launches only the kernels of one workload, steps times, for profilers."""
    import torch

    import sparse_query_attention_b200 as sqa
    from sqa_inputs import attention_inputs

    dev = torch.device("cuda", 0)
    stream = torch.cuda.current_stream(dev)
    if args.profile in ("fwd", "xsqa", "mha", "gqa"):
        w = WORKLOAD
        B, N, H_q, H_kv, d = w["B"], w["N"], w["H_q"], w["H_kv"], w["d_head"]
        if args.profile != "fwd":  # another head-count variant of the encoder workload
            H_q, H_kv = VARIANTS[{"xsqa": "xSQA", "mha": "MHA", "gqa": "GQA"}[args.profile]]
        x = attention_inputs(B, N, H_q, H_kv, d, seed=2, device=dev)
        out = torch.empty((B, N, H_q * d), dtype=torch.float32, device=dev)
        for _ in range(args.steps):
            sqa.sqa_attn_fwd(x["q"], x["k"], x["v"], out, B, N, H_q, H_kv, d, w["causal"], 1 / math.sqrt(d),
                             stream=stream)
    elif args.profile == "gemm":
        c = PROJ
        x, w = proj_operands(torch, dev)
        y = torch.empty((c["M"], c["N"]), dtype=torch.bfloat16, device=dev)
        for _ in range(args.steps):
            sqa.sqa_proj(x, w, None, y, sqa.SQA_DT_BF16, c["M"], c["K"], c["N"], stream=stream)
    elif args.profile == "decode":
        c = DECODE
        B, L, n_new, d = c["B"], c["L"], c["n_new"], c["d_head"]
        hq, hkv = DECODE_VARIANTS["SQA"]
        g = torch.Generator(device=dev)
        g.manual_seed(5)
        q = torch.randn((B, n_new, hq, d), generator=g, device=dev).to(torch.bfloat16)
        kc = torch.randn((B, L, hkv, d), generator=g, device=dev).to(torch.bfloat16)
        vc = torch.randn((B, L, hkv, d), generator=g, device=dev).to(torch.bfloat16)
        lens = torch.full((B,), L, dtype=torch.int32, device=dev)
        out = torch.empty((B, n_new, hq, d), dtype=torch.bfloat16, device=dev)
        wsb = sqa.sqa_attn_decode_workspace_size(B, n_new, hq, hkv, d, L)
        ws = torch.empty(max(wsb, 1), dtype=torch.uint8, device=dev)
        for _ in range(args.steps):
            sqa.sqa_attn_decode(q, kc, vc, lens, out, sqa.SQA_DT_BF16, None, B, n_new, hq, hkv, d, L,
                                1 / math.sqrt(d), ws if wsb else None, wsb, stream=stream)
    elif args.profile == "layer":
        layer, layer_backward = decoder_layer_step(sqa, torch, stream, dev, "SQA")
        for _ in range(args.steps):
            layer()
            layer_backward()
    elif args.profile == "memattn":
        from sqa_inputs import cross_attention_inputs
        hq, hkv, d = 8, 4, 128
        sc = 1 / math.sqrt(d)
        BF = sqa.SQA_DT_BF16
        # A short key sequence (dK/dV split) and few queries (forward and dQ
        # split), forward and backward each, bf16 in and out.
        for Nq, Nkv in ((32768, 1024), (1024, 32768)):
            x = cross_attention_inputs(1, Nq, Nkv, hq, hkv, d, seed=3, with_dout=True, device=dev)
            o = torch.empty((1, Nq, hq, d), dtype=torch.bfloat16, device=dev)
            lse = torch.empty((1, hq, Nq), dtype=torch.float32, device=dev)
            g = [torch.empty(t.shape, dtype=torch.bfloat16, device=dev) for t in (x["q"], x["k"], x["v"])]
            wsb = sqa.sqa_attn_bwd_workspace_size(1, Nq, hq, hkv, d)
            ws = torch.empty(wsb, dtype=torch.uint8, device=dev)
            for _ in range(args.steps):
                sqa.sqa_attn_fwd_cross(x["q"], x["k"], x["v"], o, BF, lse, 1, Nq, Nkv, hq, hkv, d, sc, stream=stream)
                sqa.sqa_attn_bwd_cross(x["q"], x["k"], x["v"], o, BF, x["do"], lse, g[0], g[1], g[2], BF, 1, Nq, Nkv,
                                       hq, hkv, d, sc, ws, wsb, stream=stream)
    else:
        flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
        time_training_step(sqa, torch, stream, flush, dev, reps=max(1, args.steps - 3))
    torch.cuda.synchronize(dev)
    sqa.sqa_device_status(stream)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["sqa", "reference"], default="sqa")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--profile", choices=["fwd", "xsqa", "mha", "gqa", "bwd", "decode", "gemm", "layer", "memattn"],
                    default=None,
                    help="only launch the kernels (for ncu): fwd = the bench workload's forward, "
                         "xsqa / mha / gqa = its xSQA (4,4), MHA (16,16) or GQA (16,4) variant, "
                         "gemm = the M=32768, N=K=4096 projection GEMM, "
                         "bwd = the B=4, N=8192 causal training step, decode = one SQA decode step of "
                         "B=16 sequences x 32768 cached tokens, layer = the SQA decoder-layer training "
                         "step (B=16, N=1024, d_model=256), memattn = SQA cross attention forward and "
                         "backward at 32768 queries x 1024 keys and 1024 x 32768; no timing, no JSON")
    args = ap.parse_args(argv)
    if args.profile:
        return run_profile(args)
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps
    if args.impl == "reference":
        return run_reference(args)
    return run_sqa(args)


if __name__ == "__main__":
    sys.exit(main())
