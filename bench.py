"""Benchmark: decode-attention KV GB/s (% of B200 HBM peak) and tokens/s per KV dtype.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

A step is one pass of the hot path over one batch: quantize-append of one new token per
sequence, then split-KV decode attention (+ log-sum-exp merge) over the whole cache. The
default workload is the Llama-3-8B-shaped FP8 E4M3 layer (batch 32, 32/8 heads, context
4096). Inputs are seeded synthetic tensors resident in HBM; the step is captured once in a
CUDA graph and replayed; L2 is flushed (256 MiB written, then 256 MiB read) before every timed step; the
flush is outside the step's CUDA-event interval. `value` is the step's algorithmic bytes
(codes + scales + residual + Q + out for decode, new K/V in + codes out for the append)
divided by the step time, summed over all ranks (weak scaling: one full workload per GPU).
`--impl reference` times the CPU oracle on a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "decode-attn KV GB/s (% of B200 HBM peak) and tokens/s, per KV dtype"
UNIT = "GB/s"
FALLBACK_HBM_GBS = 6650.0
DTYPE_NAME = {synth.FP8_E4M3_PER_TENSOR: "fp8_e4m3", synth.FP8_E5M2_PER_TENSOR: "fp8_e5m2", synth.INT8_SYM_PER_TENSOR: "int8",
              synth.INT8_SYM_PER_TOKEN: "int8", synth.INT8_SYM_PER_CHANNEL: "int8",
              synth.UINT8_ASYM_PER_CHANNEL: "uint8", synth.KIVI_INT4: "int4", synth.KIVI_INT2: "int2",
              synth.KIVI_INT4_F16: "int4 (fp16 meta)", synth.KIVI_INT2_F16: "int2 (fp16 meta)",
              synth.INT4_SYM_PER_GROUP: "int4"}
CALIBRATED = (synth.FP8_E4M3_PER_TENSOR, synth.FP8_E5M2_PER_TENSOR, synth.INT8_SYM_PER_TENSOR, synth.INT8_SYM_PER_CHANNEL,
              synth.UINT8_ASYM_PER_CHANNEL)
KERNEL_SOURCES = ["decode_attention_quantize_b200/csrc/kvq_decode.cu",
                  "decode_attention_quantize_b200/csrc/kvq_device.cuh"]


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="fp8_8b", choices=list(synth.workloads()))
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-per-config", action="store_true", help="measure the headline workload only")
    ap.add_argument("--batch", type=int, default=0,
                    help="run the workload with this batch instead of its own (a reduced case for profiling)")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    return ap.parse_args()


# ---------------------------------------------------------------- algorithmic bytes
def row_bytes(scheme):
    return 128 * {synth.KIVI_INT4: 4, synth.KIVI_INT2: 2, synth.INT4_SYM_PER_GROUP: 4, synth.KIVI_INT4_F16: 4,
                  synth.KIVI_INT2_F16: 2}.get(scheme, 8) // 8


def meta_bytes_per_token(scheme, Hkv, group=32):
    """Per-token-row metadata bytes that decode must read (K or V side)."""
    if scheme == synth.INT8_SYM_PER_TOKEN:
        return 4.0
    if scheme in (synth.KIVI_INT4, synth.KIVI_INT2):
        return 8.0 * 128 / 32  # fp32 (scale, min) per 32 elements
    if scheme in (synth.KIVI_INT4_F16, synth.KIVI_INT2_F16):
        return 4.0 * 128 / 32  # fp16 (scale, min) per 32 elements
    if scheme == synth.INT4_SYM_PER_GROUP:
        return 4.0 * 128 / group  # fp32 scale per group of channels
    return 0.0


def fixed_meta_bytes(scheme, Hkv):
    if scheme in (synth.FP8_E4M3_PER_TENSOR, synth.FP8_E5M2_PER_TENSOR, synth.INT8_SYM_PER_TENSOR):
        return 4
    if scheme == synth.INT8_SYM_PER_CHANNEL:
        return Hkv * 128 * 4
    if scheme == synth.UINT8_ASYM_PER_CHANNEL:
        return Hkv * 128 * 5
    return 0


def decode_bytes(w, lens_q, len_res=0):
    """Algorithmic bytes of one decode call: codes + metadata + residual + Q + out."""
    rows = int(np.sum(lens_q)) * w.Hkv
    b = rows * (row_bytes(w.k_scheme) + row_bytes(w.v_scheme))
    b += rows * (meta_bytes_per_token(w.k_scheme, w.Hkv, w.group) + meta_bytes_per_token(w.v_scheme, w.Hkv, w.group))
    b += fixed_meta_bytes(w.k_scheme, w.Hkv) + fixed_meta_bytes(w.v_scheme, w.Hkv)
    b += w.B * w.Hkv * len_res * 128 * 2 * 2
    b += w.B * w.Hq * 128 * (2 if w.bf16 else 4)  # Q
    b += w.B * w.Hq * 128 * 4                       # out (fp32)
    return float(b)


def append_bytes(w, n=1):
    """One token per sequence: read bf16/fp32 K and V, write codes (+ per-token scales)."""
    rows = w.B * w.Hkv * n
    elem = 2 if w.bf16 else 4
    b = rows * 128 * elem * 2
    if w.kivi:
        b += rows * 128 * 2 * 2  # bf16 residual write
    else:
        b += rows * (row_bytes(w.k_scheme) + row_bytes(w.v_scheme))
        b += rows * (meta_bytes_per_token(w.k_scheme, w.Hkv, w.group) + meta_bytes_per_token(w.v_scheme, w.Hkv, w.group))
    return float(b)


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as fh:
            v = float(json.load(fh)["hbm_gbs"])
            return v, "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def kernel_traffic(workload):
    """DRAM bytes per decode launch from the committed ncu capture, if the kernel source is
    unchanged since the capture; else None."""
    path = os.path.join(ROOT, "profiles", f"decode_{workload}_traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as fh:
        rec = json.load(fh)
    h = hashlib.sha256()
    for src in KERNEL_SOURCES:
        h.update(open(os.path.join(ROOT, src), "rb").read())
    if rec.get("kernel_source_sha256") != h.hexdigest():
        return None
    return rec.get("dram_bytes_per_launch_full")


# ---------------------------------------------------------------- clocks (NVML, read-only)
class ClockSampler:
    def __init__(self, index):
        self.index = index
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._t = None
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
        except Exception:
            self.nv = None

    def _run(self):
        nv = self.nv
        names = {
            getattr(nv, "nvmlClocksEventReasonHwSlowdown", 0x8): "hw_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwThermalSlowdown", 0x20): "sw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonHwThermalSlowdown", 0x40): "hw_thermal_slowdown",
            getattr(nv, "nvmlClocksEventReasonSwPowerCap", 0x4): "sw_power_cap",
            getattr(nv, "nvmlClocksEventReasonHwPowerBrakeSlowdown", 0x80): "hw_power_brake_slowdown",
        }
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                mask = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                for bit, name in names.items():
                    if mask & bit:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(0.005)

    def __enter__(self):
        if self.nv:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._t:
            self._t.join()

    def summary(self):
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                "samples": len(self.samples), "source": "nvml" if self.nv else "unavailable"}


class L2Flush:
    """Evicts the 126 MB L2 between timed steps: writes a 256 MiB buffer, then reads another
    256 MiB buffer so the write-backs of the first happen before the timed interval and the
    timed step starts with clean lines that hold none of its inputs."""

    def __init__(self, dev):
        import torch
        self.a = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.b = torch.ones(64 << 20, dtype=torch.float32, device=dev)
        self.out = torch.empty((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.a.zero_()
        torch.amax(self.b, dim=0, out=self.out)


# ---------------------------------------------------------------- multi-rank plumbing
def rank_workload(w, rank):
    """Weak scaling: rank r runs the whole per-GPU workload on its own seeded batch."""
    return synth.Workload(**{**w.__dict__, "seed": w.seed + 1000 * rank})


def max_over_ranks(seconds, world, device=None):
    """Slowest rank's timed interval (the job's time); a no-op for one process."""
    if world <= 1:
        return float(seconds)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(seconds)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(step_bytes, steps, t_max_total, world):
    """Whole-job GB/s: every rank processed `steps` steps of `step_bytes` in t_max_total."""
    return world * step_bytes * steps / t_max_total / 1e9


# ---------------------------------------------------------------- GPU workload
class GpuWorkload:
    """Builds one layer's cache for a workload and exposes a graph-captured decode step."""

    def __init__(self, w, rank, device):
        import torch
        from decode_attention_quantize_b200 import kvq
        self.torch, self.kvq, self.w, self.dev = torch, kvq, w, device
        self.seed_w = rank_workload(w, rank)
        W = self.seed_w
        if W.paged:
            self._build_paged(W)
        else:
            self._build_dense(W)
        torch.cuda.synchronize()

    def _dev(self, a, bf16):
        t = self.torch.from_numpy(np.ascontiguousarray(a)).to(self.dev)
        return t.view(self.torch.bfloat16) if bf16 else t

    def _build_dense(self, W):
        kvq = self.kvq
        total = W.prefill_tokens()
        self.append_token = W.name != "tiny_int8"  # the tiny configuration decodes without appending
        pre = total - 1 if self.append_token else total
        cap = (total + 127) // 128 * 128
        spec = kvq.CacheSpec(W.B, W.Hq, W.Hkv, W.k_scheme, W.v_scheme, capacity=cap, rotate=W.rotate, group=W.group,
                             rope_theta=W.prerope_theta)
        self.cache = kvq.QuantizedKVCache(spec, device=self.dev)
        self.calib = W.k_scheme in CALIBRATED or W.v_scheme in CALIBRATED
        self.pre_k = self._dev(synth.keys(W, 0, W.B, 0, W.Hkv, 0, pre), W.bf16)
        self.pre_v = self._dev(synth.values(W, 0, W.B, 0, W.Hkv, 0, pre), W.bf16)
        self.pre_lens = None
        self.cache.append(self.pre_k, self.pre_v, calibrate=self.calib)
        self.torch.cuda.synchronize()
        self.pre = pre
        self.prefill_rows = W.B * W.Hkv * pre
        d = self.cache.desc
        self.saved = (d.num_quantized, d.num_residual)
        self.k_new = self._dev(synth.keys(W, 0, W.B, 0, W.Hkv, pre, pre + 1), W.bf16)
        self.v_new = self._dev(synth.values(W, 0, W.B, 0, W.Hkv, pre, pre + 1), W.bf16)
        self._common(W)

    def reset_to_empty(self):
        """Forget every token (dense: host lengths; paged: device lengths) so the prefill can be
        appended again onto the same positions."""
        d = self.cache.desc
        if self.w.paged:
            self.cache["seq_lens"].zero_()
        else:
            d.num_quantized, d.num_residual = 0, 0

    def prefill_bytes(self, reads=None):
        """Algorithmic bytes of the prefill append: the block is read once (twice when it
        calibrates a per-tensor / per-channel scale: the 2R + W count; reads=1 gives R + W) and
        codes, metadata and residual written."""
        W = self.seed_w
        rows = self.prefill_rows
        elem = 2 if W.bf16 else 4
        if reads is None:
            reads = 2 if self.calib else 1
        b = rows * 128 * elem * 2 * reads
        if W.kivi:
            nq = (self.cache.desc.num_quantized if not W.paged else 0)
            qrows = W.B * W.Hkv * nq
            b += qrows * (row_bytes(W.k_scheme) + row_bytes(W.v_scheme))
            b += qrows * (meta_bytes_per_token(W.k_scheme, W.Hkv) + meta_bytes_per_token(W.v_scheme, W.Hkv))
            b += W.B * W.Hkv * self.cache.desc.num_residual * 128 * 2 * 2
        else:
            b += rows * (row_bytes(W.k_scheme) + row_bytes(W.v_scheme))
            b += rows * (meta_bytes_per_token(W.k_scheme, W.Hkv, W.group) + meta_bytes_per_token(W.v_scheme, W.Hkv, W.group))
        return float(b)

    def time_prefill(self, flush, stream, reps=3):
        torch = self.torch
        ms = []
        saved = (self.cache.desc.num_quantized, self.cache.desc.num_residual)
        for _ in range(reps):
            self.reset_to_empty()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                flush()
                a.record(stream)
                self.cache.append(self.pre_k, self.pre_v, new_lens=self.pre_lens, calibrate=self.calib,
                                  stream=stream)
                b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        if not self.w.paged:
            self.cache.desc.num_quantized, self.cache.desc.num_residual = saved
        return sum(ms) / len(ms) / 1e3

    def time_rescale(self, flush, stream, reps=3):
        """Rescaling append of one token per sequence whose values are 2^(i+1) times the step
        token's, so every repetition grows the batch-wide scales and requantizes every cached
        code. Dense caches with batch-wide scales only; leaves the cache rescaled."""
        torch = self.torch
        d = self.cache.desc
        ms = []
        for i in range(reps):
            f = float(2 ** (i + 1))
            k = (self.k_new.float() * f).to(self.k_new.dtype)
            v = (self.v_new.float() * f).to(self.v_new.dtype)
            d.num_quantized, d.num_residual = self.saved
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            with torch.cuda.stream(stream):
                flush()
                a.record(stream)
                self.cache.append(k, v, rescale=True, stream=stream)
                b.record(stream)
            torch.cuda.synchronize()
            ms.append(a.elapsed_time(b))
        W = self.seed_w
        cached = W.B * W.Hkv * self.saved[0]
        nbytes = 0.0
        for sch in (W.k_scheme, W.v_scheme):
            if sch in CALIBRATED:
                nbytes += 2.0 * cached * row_bytes(sch)  # every cached code read and written
        nbytes += 2 * (W.B * W.Hkv * 128 * (2 if W.bf16 else 4)) * 2  # the token, read twice
        nbytes += W.B * W.Hkv * (row_bytes(W.k_scheme) + row_bytes(W.v_scheme))
        return sum(ms) / len(ms) / 1e3, nbytes, cached

    def _build_paged(self, W):
        kvq, torch = self.kvq, self.torch
        lens = W.prefill_lengths()
        extra = 4096
        need = [(int(L) + extra + W.page_size - 1) // W.page_size for L in lens]
        max_pages = max(need)
        num_pages = int(sum(need))
        perm = synth.permutation(W.seed, num_pages)
        table = np.full((W.B, max_pages), -1, np.int32)
        off = 0
        for b, n in enumerate(need):
            table[b, :n] = perm[off:off + n]
            off += n
        spec = kvq.CacheSpec(W.B, W.Hq, W.Hkv, W.k_scheme, W.v_scheme, paged=True, page_size=W.page_size,
                             max_pages=max_pages, num_pages=num_pages, rotate=W.rotate, group=W.group)
        self.cache = kvq.QuantizedKVCache(spec, device=self.dev, page_table=torch.from_numpy(table))
        n_max = int(lens.max())
        K = torch.zeros((W.B, W.Hkv, n_max, 128), dtype=torch.bfloat16, device=self.dev)
        V = torch.zeros_like(K)
        for b in range(W.B):
            L = int(lens[b])
            K[b, :, :L] = self._dev(synth.keys(W, b, b + 1, 0, W.Hkv, 0, L)[0], True)
            V[b, :, :L] = self._dev(synth.values(W, b, b + 1, 0, W.Hkv, 0, L)[0], True)
        self.pre_k, self.pre_v = K, V
        self.pre_lens = torch.from_numpy(lens).to(self.dev)
        self.calib = True
        self.prefill_rows = int(lens.sum()) * W.Hkv
        self.cache.append(K, V, new_lens=self.pre_lens, calibrate=True)
        torch.cuda.synchronize()
        self.lens = lens
        self.append_token = True
        self.extra = extra
        # step tokens: generated per step index from the same generator (positions L_b + s)
        self.k_steps, self.v_steps = [], []
        self._common(W)

    def _common(self, W):
        torch, kvq = self.torch, self.kvq
        self.q_host = [synth.queries(W, s, 0, W.B) for s in range(2)]
        self.q = self._dev(self.q_host[0], W.bf16)
        self.out = torch.empty((W.B, W.Hq, 128), dtype=torch.float32, device=self.dev)
        self.ws = kvq.decode_workspace(self.cache.desc, self.dev)
        self.scale = 1.0 / math.sqrt(128.0)

    def paged_token(self, step):
        W = self.seed_w
        k = np.stack([synth.keys(W, b, b + 1, 0, W.Hkv, int(self.lens[b]) + step, int(self.lens[b]) + step + 1)[0]
                      for b in range(W.B)])
        v = np.stack([synth.values(W, b, b + 1, 0, W.Hkv, int(self.lens[b]) + step, int(self.lens[b]) + step + 1)[0]
                      for b in range(W.B)])
        return self._dev(k, True), self._dev(v, True)

    # one step (eager): append + decode, through the library's one-call step (the decode of a
    # dense 8-bit / INT4 cache then reads the cached tiles while the append runs)
    def step(self, stream=None, k_new=None, v_new=None, q=None):
        d = self.cache.desc
        q = self.q if q is None else q
        if self.append_token:
            if not self.w.paged:
                d.num_quantized, d.num_residual = self.saved
            self.cache.append_decode(self.k_new if k_new is None else k_new, self.v_new if v_new is None else v_new,
                                     q, self.scale, out=self.out, workspace=self.ws, stream=stream)
        else:
            self.cache.decode(q, self.scale, out=self.out, workspace=self.ws, stream=stream)

    def decode_lens(self, appended):
        """(per-sequence quantized tokens, residual tokens) seen by a decode. Dense: every step
        sees the state after its own append (recorded after the first step). Paged: the cache
        holds the prefill plus `appended` streamed tokens."""
        W = self.seed_w
        if W.paged:
            return self.lens + appended, 0
        nq, nr = self.after
        return np.full(W.B, nq), (nr if W.kivi else 0)


def measure_workload(name, rank, world, dev, steps, warmup, stream, flush, e2e=True):
    """Build one workload's cache, time its bulk prefill append, then `steps` graph-replayed
    steps (append + decode) and up to 400 decode calls, L2 flushed before each; device time by
    CUDA events on the launching stream."""
    import torch
    import torch.distributed as dist
    from decode_attention_quantize_b200 import kvq
    w = synth.workloads()[name]
    G = GpuWorkload(w, rank, dev)
    W = G.seed_w
    t_prefill = G.time_prefill(flush, stream)
    prefill = {"ms": t_prefill * 1e3, "bytes": G.prefill_bytes(), "bytes_r_plus_w": G.prefill_bytes(reads=1),
               "tokens": G.prefill_rows // W.Hkv, "calibrating": bool(G.calib)}
    G.pre_k = G.pre_v = None  # release the prefill block before timing the steps
    torch.cuda.empty_cache()

    # capture one step in a CUDA graph (dense: positions are reset each step, so the graph
    # replays an identical step; paged: lengths live on the device and advance per replay)
    graph = None
    launches_per_replay = 0
    if not W.paged:
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            G.step(stream)  # materialise lazy state before capture
        torch.cuda.synchronize()
        G.after = (G.cache.desc.num_quantized, G.cache.desc.num_residual)
        graph = torch.cuda.CUDAGraph()
        c0 = kvq.kvq_launch_count()
        with torch.cuda.graph(graph, stream=stream):
            G.step(stream)
        launches_per_replay = kvq.kvq_launch_count() - c0  # kernels in the captured step
        torch.cuda.synchronize()

    def run_step(i):
        graph.replay()

    # paged: pre-generate the step tokens (host generation is outside timing)
    if W.paged:
        total_steps = warmup + steps
        if total_steps + 200 > G.extra:
            raise SystemExit("too many steps for the page pool")
        toks = [G.paged_token(i) for i in range(total_steps)]

        def run_step(i):  # noqa: F811
            with torch.cuda.stream(stream):
                G.step(stream, k_new=toks[i][0], v_new=toks[i][1])

    for i in range(warmup):
        flush()
        run_step(i)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    launches0 = kvq.kvq_launch_count()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        with torch.cuda.stream(stream):
            flush()
            ev[i][0].record(stream)
            run_step(warmup + i)
            ev[i][1].record(stream)
    torch.cuda.synchronize()
    step_ms = [a.elapsed_time(b) for a, b in ev]
    launches = kvq.kvq_launch_count() - launches0
    if graph is not None:
        launches = steps * launches_per_replay
    # decode-only timing (the dominant kernel's call: split-KV kernel + merge), eager
    n_dec = min(steps, 400)
    dec_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(n_dec)]
    for i in range(n_dec):
        with torch.cuda.stream(stream):
            flush()
            dec_ev[i][0].record(stream)
            G.cache.decode(G.q, G.scale, out=G.out, workspace=G.ws, stream=stream)
            dec_ev[i][1].record(stream)
    torch.cuda.synchronize()
    dec_ms = [a.elapsed_time(b) for a, b in dec_ev]

    t_step = sum(step_ms) / len(step_ms) / 1e3  # seconds (mean)
    t_dec = sum(dec_ms) / len(dec_ms) / 1e3
    lens_q, len_res = G.decode_lens(warmup + steps // 2 + 1)
    dbytes = decode_bytes(W, lens_q, len_res)
    lens_d, res_d = G.decode_lens(warmup + steps)  # state seen by the decode-only timing
    dbytes_dec = decode_bytes(W, lens_d, res_d)
    abytes = append_bytes(W) if G.append_token else 0.0
    t_max = max_over_ranks(sum(step_ms) / 1e3, world, device=dev) / steps

    # end to end through the public API: host inputs (pinned) -> device -> step -> host out
    e2e_r = run_e2e(G, W, stream, flush, n=min(200, steps), step0=warmup + steps) if e2e else None
    status = G.cache.status()
    return dict(t_step=t_step, t_max=t_max, t_dec=t_dec, dbytes=dbytes, dbytes_dec=dbytes_dec, abytes=abytes,
                launches=launches, prefill=prefill, e2e=e2e_r, status=status, W=W, G=G)


# every workload the library measures; the headline line is `--workload`, the rest go into
# `per_config` (one process, one GPU, shorter runs)
PER_CONFIG = ["tiny_int8", "fp8_8b", "e5m2_8b", "fp8_8b_prerope", "kivi4_70b", "kivi4f16_70b", "int4g_70b",
              "int4g_rot_70b", "int4g128_70b", "kivi2_131k", "kivi2f16_131k", "paged_int8"]
NOMINAL_HBM_GBS = 8000.0  # the ~8 TB/s B200 figure the targets are stated against


def config_summary(r, peak):
    """One workload's line of `per_config`: the decode call, the step and the bulk append."""
    W = r["W"]
    gbs = r["dbytes_dec"] / r["t_dec"] / 1e9
    pf = r["prefill"]
    t_pf = pf["ms"] / 1e3
    return {"workload": W.name, "dtype": dtype_of(W), "layout": "paged/16" if W.paged else "dense",
            "decode_ms": r["t_dec"] * 1e3, "decode_GBps": gbs, "frac": gbs / peak,
            "frac_nominal_8TBps": gbs / NOMINAL_HBM_GBS, "algorithmic_bytes": r["dbytes_dec"],
            "traffic": kernel_traffic(W.name), "step_ms": r["t_step"] * 1e3, "tokens_per_s": W.B / r["t_step"],
            "append_bulk": {"ms": pf["ms"], "calibrating": pf["calibrating"],
                            "GBps_2R_plus_W": pf["bytes"] / t_pf / 1e9, "frac_2R_plus_W": pf["bytes"] / t_pf / 1e9 / peak,
                            "GBps_R_plus_W": pf["bytes_r_plus_w"] / t_pf / 1e9,
                            "frac_R_plus_W": pf["bytes_r_plus_w"] / t_pf / 1e9 / peak},
            "device_status": list(r["status"])}


def run_gpu(args, rank, world, local_rank):
    import torch
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    stream = torch.cuda.Stream(device=dev)
    flush = L2Flush(dev)
    sampler = ClockSampler(local_rank)  # samples the whole GPU section, every workload
    with sampler:
        r = measure_workload(args.workload, rank, world, dev, args.steps, args.warmup, stream, flush)
        per_config = None
        if world == 1 and not args.no_per_config:
            peak, _ = measured_peak()
            per_config = []
            for name in PER_CONFIG:
                if name == args.workload:
                    per_config.append(config_summary(r, peak))
                    continue
                rc = measure_workload(name, rank, world, dev, min(args.steps, 30), 3, stream, flush, e2e=False)
                per_config.append(config_summary(rc, peak))
                del rc
                torch.cuda.empty_cache()
        torch.cuda.synchronize()
    r["clocks"] = sampler.summary()
    r["per_config"] = per_config
    return r


def run_e2e(G, W, stream, flush, n, step0):
    """Same step through the public API with host buffers: pinned host K/V token and Q copied
    in, append + decode, output copied back; all inside the event interval."""
    import torch
    torch_dt = torch.bfloat16 if W.bf16 else torch.float32
    q_h = torch.from_numpy(np.ascontiguousarray(G.q_host[1])).view(torch_dt).pin_memory()
    if W.paged:
        toks = [G.paged_token(step0 + i) for i in range(n)]
        k_h = [t[0].cpu().pin_memory() for t in toks]
        v_h = [t[1].cpu().pin_memory() for t in toks]
    else:
        k_h = [G.k_new.detach().cpu().pin_memory()] * n
        v_h = [G.v_new.detach().cpu().pin_memory()] * n
    out_h = torch.empty(G.out.shape, dtype=torch.float32).pin_memory()
    q_d = torch.empty_like(G.q)
    kd = torch.empty_like(k_h[0], device=G.dev)
    vd = torch.empty_like(v_h[0], device=G.dev)
    h2d = q_h.numel() * q_h.element_size()
    if G.append_token:
        h2d += 2 * k_h[0].numel() * k_h[0].element_size()
    d2h = out_h.numel() * 4
    evs = []
    for i in range(n):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            flush()
            a.record(stream)
            q_d.copy_(q_h, non_blocking=True)
            if G.append_token:
                kd.copy_(k_h[i], non_blocking=True)
                vd.copy_(v_h[i], non_blocking=True)
            G.step(stream, k_new=kd, v_new=vd, q=q_d)
            out_h.copy_(G.out, non_blocking=True)
            b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    ms = sum(a.elapsed_time(b) for a, b in evs) / n
    return dict(t=ms / 1e3, h2d=h2d, d2h=d2h)


# ---------------------------------------------------------------- quantization error
def _rope_rows(K, theta):
    """Rotate-half RoPE of key rows K [T, 128] at positions 0..T-1 (fp64), for the error reference
    of caches that hold keys before RoPE."""
    T, D = K.shape
    inv = theta ** (-2.0 * np.arange(D // 2) / D)
    ang = np.arange(T)[:, None] * inv[None, :]
    c, s = np.cos(ang), np.sin(ang)
    a, b = K[:, :D // 2], K[:, D // 2:]
    return np.concatenate([a * c - b * s, b * c + a * s], axis=1)


def _f64(a, bf16):
    a = np.asarray(a)
    if bf16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def quant_error(G, W, stream, n_pairs=8):
    """Quantization error of the step's output: the library's decode of the final cache state
    against fp64 attention over the unquantized inputs the cache was built from, on sampled
    (sequence, kv head) pairs; dense caches also report the per-element error of the
    dequantized K and V of those pairs. Informational (not a parity check)."""
    import torch
    d = G.cache.desc
    with torch.cuda.stream(stream):
        G.cache.decode(G.q, G.scale, out=G.out, workspace=G.ws, stream=stream)
    torch.cuda.synchronize()
    out = G.out.cpu().numpy().astype(np.float64)
    if W.paged:
        lens = G.cache["seq_lens"].cpu().numpy().astype(np.int64)
    else:
        lens = np.full(W.B, d.num_quantized + (d.num_residual if W.kivi else 0), np.int64)
    allp = [(b, h) for b in range(W.B) for h in range(W.Hkv)]
    rng = np.random.default_rng(W.seed + 99)
    pairs = [allp[i] for i in sorted(rng.choice(len(allp), size=min(n_pairs, len(allp)), replace=False))]
    q = _f64(G.q_host[0], W.bf16)
    scale = float(np.float32(G.scale))
    diffs, refs, kd, kx, vd, vx = [], [], [], [], [], []
    deq = None if W.paged else [G.cache.dequantize(which, int(lens[0])) for which in (0, 1)]
    torch.cuda.synchronize()
    for b, h in pairs:
        L = int(lens[b])
        K = _f64(synth.keys(W, b, b + 1, h, h + 1, 0, L)[0, 0], W.bf16)
        V = _f64(synth.values(W, b, b + 1, h, h + 1, 0, L)[0, 0], W.bf16)
        qs = q[b, h * W.G:(h + 1) * W.G]
        Kr = _rope_rows(K, W.prerope_theta) if W.prerope_theta > 0 else K
        sc = qs @ Kr.T * scale
        pr = np.exp(sc - sc.max(axis=1, keepdims=True))
        ref = (pr @ V) / pr.sum(axis=1, keepdims=True)
        diffs.append(out[b, h * W.G:(h + 1) * W.G] - ref)
        refs.append(ref)
        if deq is not None:
            kd.append(deq[0][b, h, :L].cpu().numpy().astype(np.float64) - K)
            kx.append(K)
            vd.append(deq[1][b, h, :L].cpu().numpy().astype(np.float64) - V)
            vx.append(V)
    dd, rr = np.concatenate([x.ravel() for x in diffs]), np.concatenate([x.ravel() for x in refs])
    res = {"vs": "fp64 attention over the unquantized inputs (same tokens, same queries)",
           "pairs": len(pairs), "max_abs": float(np.abs(dd).max()),
           "max_abs_rel": float(np.abs(dd).max() / np.abs(rr).max()),
           "rel_l2": float(np.linalg.norm(dd) / np.linalg.norm(rr)),
           "clamped_elements": int(G.cache.status()[1])}
    if deq is not None:
        for name, dl, xl in (("k", kd, kx), ("v", vd, vx)):
            e, x = np.concatenate([a.ravel() for a in dl]), np.concatenate([a.ravel() for a in xl])
            res[f"{name}_dequant_rel_l2"] = float(np.linalg.norm(e) / np.linalg.norm(x))
            res[f"{name}_dequant_max_abs"] = float(np.abs(e).max())
    return res


# ---------------------------------------------------------------- CPU oracle sample
class OracleUnit:
    """One (sequence, kv_head) unit of the workload held by the CPU oracle: its prefill is
    quantized once (untimed); a step is the same as on the GPU: one token appended at the
    step position, then fp64 decode attention of the unit's query heads over its tokens."""

    def __init__(self, w, b, h):
        from oracle import OracleCache
        self.w, self.b, self.h = w, b, h
        L = int(w.prefill_lengths()[b])
        self.append = w.name != "tiny_int8"
        pre = L - 1 if self.append else L
        K = synth.keys(w, b, b + 1, h, h + 1, 0, pre + 1)
        V = synth.values(w, b, b + 1, h, h + 1, 0, pre + 1)
        cap = (pre + 1 + 127) // 128 * 128
        self.oc = OracleCache(1, w.G, 1, 128, w.k_scheme, w.v_scheme, cap=cap, rotate=w.rotate, group=w.group,
                              rope_theta=w.prerope_theta)
        calib = w.k_scheme in CALIBRATED or w.v_scheme in CALIBRATED
        self.oc.append(K[:, :, :pre], V[:, :, :pre], w.bf16, calibrate=calib)
        self.saved = (self.oc.c.len, self.oc.c.res)
        self.k1, self.v1 = K[:, :, pre:pre + 1].copy(), V[:, :, pre:pre + 1].copy()
        qw = synth.Workload(**{**w.__dict__, "B": 1, "Hkv": 1, "Hq": w.G, "seed": w.seed + 17 * (b * w.Hkv + h)})
        self.q = synth.queries(qw, 0, 0, 1)
        self.unit_w = synth.Workload(**{**w.__dict__, "B": 1, "Hkv": 1, "Hq": w.G})

    def step(self):
        """Returns (algorithmic bytes, seconds) of one oracle step."""
        self.oc.c.len, self.oc.c.res = self.saved
        t0 = time.perf_counter()
        if self.append:
            self.oc.append(self.k1, self.v1, self.w.bf16)
        self.oc.decode(self.q, self.w.bf16, 1.0 / math.sqrt(128.0))
        dt = time.perf_counter() - t0
        nr = self.oc.residual if self.w.kivi else 0
        b = decode_bytes(self.unit_w, np.array([self.oc.length]), nr)
        if self.append:
            b += append_bytes(self.unit_w)
        return b, dt


_UNITS = {}


def _oracle_worker(job):
    """One process of the all-cores oracle baseline: unit `i` of the workload (built once per
    process, untimed), stepped until `seconds` of timed work. Returns (bytes, seconds, steps)."""
    name, i, seconds = job
    w = synth.workloads()[name]
    if (name, i) not in _UNITS:
        _UNITS[(name, i)] = OracleUnit(w, i % w.B, (i // w.B) % w.Hkv)
    u = _UNITS[(name, i)]
    tb = tt = 0.0
    n = 0
    while tt < seconds:
        b, t = u.step()
        tb, tt, n = tb + b, tt + t, n + 1
    return tb, tt, n


def oracle_time_all_cores(w, seconds):
    """The oracle over independent (sequence, kv_head) units, one process per host core (spawned:
    the parent has already used the GPU). The processes run concurrently, so the aggregate
    throughput is the sum of their rates over their timed work."""
    import multiprocessing as mp
    n = max(1, min(os.cpu_count() or 1, 64, w.B * w.Hkv))
    ctx = mp.get_context("spawn")
    with ctx.Pool(n) as pool:
        res = pool.map(_oracle_worker, [(w.name, i, seconds) for i in range(n)], chunksize=1)
    rate = sum(r[0] / r[1] for r in res)
    steps = sum(r[2] for r in res)
    return rate, n, f"{steps} oracle steps, {n} concurrent processes (one unit each, {seconds:.0f} s of timed work each)"


def oracle_time(w, seconds, max_units=8):
    """Time oracle steps over up to max_units distinct units until `seconds` of timed work."""
    units, tb, tt, steps = [], 0.0, 0.0, 0
    while tt < seconds:
        if len(units) < max_units:
            i = len(units)
            units.append(OracleUnit(w, i % w.B, (i // w.B) % w.Hkv))
        u = units[steps % len(units)]
        b, t = u.step()
        tb, tt, steps = tb + b, tt + t, steps + 1
    ctx = units[0].oc.length + (units[0].oc.residual if w.kivi else 0)
    desc = (f"{steps} oracle steps over {len(units)} (sequence, kv_head) units; each: "
            f"{'append 1 token + ' if units[0].append else ''}fp64 decode of {w.G} query heads over "
            f"{ctx} tokens (single-threaded C)")
    return tb, tt, steps, desc


def dtype_of(w):
    return DTYPE_NAME[w.k_scheme] + ("/" + DTYPE_NAME[w.v_scheme] if w.v_scheme != w.k_scheme else "")


def emit(obj):
    print(json.dumps(obj), flush=True)


def main():
    args = parse()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.batch:
        base = synth.workloads()[args.workload]
        synth.register_workload(synth.Workload(**{**base.__dict__, "B": args.batch}))
        args.no_per_config = True
    w = synth.workloads()[args.workload]
    dtype = dtype_of(w)
    config = {"workload": w.name, "batch": w.B, "q_heads": w.Hq, "kv_heads": w.Hkv, "head_dim": w.D,
              "k_scheme": w.k_scheme, "v_scheme": w.v_scheme,
              "context": (f"uniform {w.len_lo}..{w.len_hi}" if w.paged else w.prefill_tokens()),
              "layout": "paged/16" if w.paged else "dense",
              "rotation": "walsh-hadamard" if w.rotate else "none",
              "keys": (f"cached before RoPE, RoPE (base {w.prerope_theta:g}) applied at decode" if w.prerope_theta > 0
                       else "cached as given"),
              "group": w.group,
              "step": ("decode only" if w.name == "tiny_int8" else "append 1 token per sequence + decode"),
              "l2": "flushed before every timed step (256 MiB write, then 256 MiB read), outside the event interval",
              "parallelism": f"replicas x{args.gpus}"}
    if args.impl == "reference":
        if rank != 0:
            return
        unit = OracleUnit(w, 0, 0)
        for _ in range(args.warmup):
            unit.step()
        tb = tt = 0.0
        for _ in range(args.steps):
            b, t = unit.step()
            tb, tt = tb + b, tt + t
        val = tb / tt / 1e9
        ctx = unit.oc.length + (unit.oc.residual if w.kivi else 0)
        sample = (f"each step: one (sequence 0, kv_head 0) unit of the workload step - "
                  f"{'append 1 token + ' if unit.append else ''}fp64 decode of {w.G} query heads over {ctx} "
                  f"tokens (single-threaded C oracle)")
        emit({"impl": "reference", "metric": METRIC, "value": val, "unit": UNIT, "n_gpus": args.gpus,
              "steps": args.steps, "warmup": args.warmup, "ms_per_step": tt / args.steps * 1e3,
              "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": dtype,
              "data": "synthetic (seeded generators)", "config": config,
              "cpu_baseline": {"value": val, "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample},
              "e2e": {"value": val, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}})
        return

    import torch
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    r = run_gpu(args, rank, world, local_rank)
    W = r["W"]
    step_bytes = r["dbytes"] + r["abytes"]
    value = job_value(step_bytes, args.steps, r["t_max"] * args.steps, world)
    tokens_per_s = world * W.B / r["t_max"]
    peak, peak_kind = measured_peak()
    achieved = r["dbytes_dec"] / r["t_dec"] / 1e9
    roofline = {"bound": "hbm", "kernel": "decode attention call (split-KV kernel + LSE merge)",
                "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "peak_source": f"{peak_kind} (MEASURED_PEAKS.json hbm_gbs)" if peak_kind == "measured" else "fallback 6.65 TB/s",
                "frac_nominal_8TBps": achieved / NOMINAL_HBM_GBS,
                "algorithmic_bytes_per_launch": r["dbytes_dec"], "launch_ms": r["t_dec"] * 1e3,
                "traffic": kernel_traffic(W.name)}
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": r["t_max"] * 1e3, "higher_is_better": True,
           "scaling": "weak", "vs_baseline": None, "dtype": dtype,
           "data": "synthetic (seeded counter-based generators; no dataset)", "config": config,
           "tokens_per_s": tokens_per_s, "pct_of_hbm_peak": 100.0 * (value / world) / peak,
           "roofline": roofline, "clocks": r["clocks"], "gpu_launches": r["launches"],
           "device_status": list(r["status"])}
    pf = r["prefill"]
    pf_gbs = pf["bytes"] / (pf["ms"] / 1e3) / 1e9
    out["append_bulk"] = {"what": "prefill quantize-append of the whole context (calibrating when the scheme "
                                  "has batch-wide scales), mean of 3, L2 flushed before each",
                          "ms": pf["ms"], "algorithmic_bytes": pf["bytes"], "GBps": pf_gbs, "frac": pf_gbs / peak,
                          "count": "2R+W when calibrating (the block is read for the statistics, then to quantize)",
                          "algorithmic_bytes_r_plus_w": pf["bytes_r_plus_w"],
                          "GBps_r_plus_w": pf["bytes_r_plus_w"] / (pf["ms"] / 1e3) / 1e9,
                          "frac_r_plus_w": pf["bytes_r_plus_w"] / (pf["ms"] / 1e3) / 1e9 / peak,
                          "tokens_per_seq": pf["tokens"] if not W.paged else "variable",
                          "calibrating": pf["calibrating"]}
    if r["e2e"]:
        e = r["e2e"]
        out["e2e"] = {"value": world * step_bytes / e["t"] / 1e9, "unit": UNIT,
                      "h2d_bytes_per_step": e["h2d"], "d2h_bytes_per_step": e["d2h"]}
    else:
        out["e2e"] = None
    if rank == 0:
        out["quant_error"] = quant_error(r["G"], W, torch.cuda.current_stream())
        G = r["G"]
        if not W.paged and not W.kivi and G.calib and G.append_token:
            t_rs, b_rs, cached = G.time_rescale(L2Flush(G.dev), torch.cuda.current_stream())
            gbs = b_rs / t_rs / 1e9
            out["rescale"] = {"what": "rescaling append of one token per sequence that grows the batch-wide "
                                      "scales: every cached code requantized, mean of 3, L2 flushed before each "
                                      "(after the timed steps)",
                              "ms": t_rs * 1e3, "algorithmic_bytes": b_rs, "cached_rows": cached, "GBps": gbs,
                              "frac": gbs / peak}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        b, t, n, desc = oracle_time(W, args.cpu_seconds)
        out["cpu_baseline"] = {"value": b / t / 1e9, "unit": UNIT, "cores": 1, "kind": "oracle",
                               "sample": desc}
        rate, ncores, desc_all = oracle_time_all_cores(W, args.cpu_seconds / 2)
        out["cpu_baseline"]["all_cores"] = {"value": rate / 1e9, "unit": UNIT, "cores": ncores, "sample": desc_all}
    if r["per_config"] is not None:
        out["per_config"] = r["per_config"]
    if world > 1:
        import torch.distributed as dist
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0:
        emit(out)


if __name__ == "__main__":
    main()
