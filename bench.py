"""Benchmark of the Hadamard-rotated Q4_0 KV cache on B200.

One step = one pass of the whole hot path over one batch.  The default
workload is the long-context decode (1 sequence, 131072 tokens, 32 query /
4 kv heads, D = 256, bf16 inputs): one kvq_decode_step call -- quantize-on-
append of the new token's K and V (rotate + Q4_0 + store) and decode attention
over the whole cache including it (rotate q, stream and dequantize the
nibbles, online softmax, split-K combine, back-rotation).

`value` is HBM throughput in GB/s: algorithmic bytes per step (every cache
byte read once, inputs read and outputs written once) / device time per
step, summed over ranks.  The timed steps replay CUDA graphs of the step back
to back, as a decode loop drives it; `e2e` calls the public API eagerly with
host copies in and out.  Every workload's data is larger than the 126 MB L2;
the long-decode cache (151 MB) is additionally kept in three copies (453 MB)
that steps rotate through.  The other workloads are timed per call (with a
512 MB L2 flush before each call, outside the timed events) and reported
under "workloads"; `--workload NAME` makes one of them the main line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
                    [--workload long_decode|long_decode_q8|quantize|paged_decode|octave]
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from hadamard_rotated_bit_fwht_b200 import synth  # noqa: E402

METRIC = "Q4+FWHT decode-attn HBM GB/s (% of peak), tok*head/s; quantize Mtok/s"
HBM_NOMINAL = 8000.0


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# the sources that decide each captured kernel's code and launch shape
_COMMON = ["kvq_internal.cuh", "kvq_api.cu"]
_DECODE = _COMMON + ["decode_common.cuh", "q4_vec.cuh", "q4_decode.cu"]
TRAFFIC_SOURCES = {
    "q4_decode_long": _DECODE + ["q4_decode_mma.cu"],
    "q4_decode_paged": _DECODE + ["q4_decode_mma.cu"],
    "q8_decode_long": _DECODE + ["q8_decode_mma.cu"],
    "q4_decode_combine": _DECODE,
    "q4_append_prefill": _COMMON + ["q4_vec.cuh", "q4_quant.cu"],
    "octave_decode": _COMMON + ["octave.cu", "octave_decode_mma.cu"],
    "octave_quantize": _COMMON + ["octave_quant.cuh", "octave_quant.cu",
                                  "octave_quant_bf16_v3.cu", "octave_quant_bf16_v4.cu"],
}


def kernel_source_hash(key: str) -> str:
    """Hash of the CUDA sources behind one traffic entry."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hadamard_rotated_bit_fwht_b200", "csrc")
    for f in sorted(set(TRAFFIC_SOURCES[key])):
        h.update(f.encode() + b"\0")
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(key: str):
    """DRAM bytes per call from a committed ncu capture, only if the kernel's
    sources are unchanged since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p) or key not in TRAFFIC_SOURCES:
        return None
    e = json.load(open(p)).get(key)
    if not e or e.get("source_hash") != kernel_source_hash(key):
        return None
    return e.get("bytes_per_call")


# ----------------------------------------------------------------- ranks
def max_over_ranks(values, dist=None, device="cpu"):
    """Element-wise maximum of per-rank timings (no-op without a process
    group); every rank gets the same result."""
    if dist is None:
        return [float(v) for v in values]
    import torch
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


def job_throughput_gbs(bytes_per_step_per_rank, world, ms_per_step):
    """Whole-job GB/s: every rank processes its own replica of the step; the
    job's step time is the slowest rank's."""
    return bytes_per_step_per_rank * world / ms_per_step / 1e6


# ----------------------------------------------------------------- clocks
class ClockSampler:
    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, val in zip(names, f[5:9]):
                if val.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ----------------------------------------------------------------- workloads
def bf16_tensor(a, dev):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).view(torch.bfloat16).to(dev)


class Workload:
    """One step of the hot path on a synthetic batch: pre(i) (the append of
    the step's new tokens, if any) then kernel_call(i) (the dominant call).
    Subclasses set step_bytes / kernel_bytes (algorithmic), launches_per_step,
    kernel_name, traffic_key, config, and for e2e the names of the step's
    input tensors (h2d) and the output tensors (d2h)."""
    launches_per_step = 0
    kernel_name = ""
    traffic_key = ""
    cycle = 1  # steps rotate through this many input copies

    def pre(self, i):
        pass

    def kernel_call(self, i):
        raise NotImplementedError

    def step(self, i):
        self.pre(i)
        self.kernel_call(i)

    def extra(self, call_ms):
        return {}


class LongDecode(Workload):
    """Long-context decode step: append the new token and decode over all
    131072 tokens in one kvq_decode_step call (the split holding the new
    position quantizes it in its prologue)."""
    launches_per_step = 2  # decode split (with the append) + combine
    kernel_name = "kvq_decode_step (q4_decode_mma_kernel with append + q4_decode_combine_kernel)"
    traffic_key = "q4_decode_long"

    bits = 4

    def __init__(self, dev, copies=3):
        import torch
        from hadamard_rotated_bit_fwht_b200 import kvq
        W = synth.WORKLOADS["long_decode"]
        B, H, T, Hq = W["batch"], W["n_kv_heads"], W["ctx"], W["n_q_heads"]
        self.B, self.H, self.T, self.Hq = B, H, T, Hq
        k, v = synth.kv_tokens(W["seed"], B, T, H, 256, W["outlier_frac"], W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        del k, v
        kd, vd = bf16_tensor(kb, dev), bf16_tensor(vb, dev)
        self.caches = []
        zero = torch.zeros(B, dtype=torch.int32, device=dev)
        self.cycle = copies
        for _ in range(copies):
            c = kvq.Q4Cache.contiguous(B, H, T, device=dev, bits=self.bits)
            kvq.quantize_append(c, kd, vd, zero)
            self.caches.append(c)
        del kd, vd
        self.q = bf16_tensor(synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256)), dev)
        self.new_k = bf16_tensor(kb[:, T - 1], dev)  # [B, Hkv, 256]
        self.new_v = bf16_tensor(vb[:, T - 1], dev)
        self.pos = torch.full((B,), T - 1, dtype=torch.int32, device=dev)
        self.lens = torch.full((B,), T, dtype=torch.int32, device=dev)
        self.out = torch.empty((B, Hq, 256), dtype=torch.float32, device=dev)
        self.ws = torch.empty(kvq.decode_attn_workspace(self.caches[0], B, Hq, T),
                              dtype=torch.uint8, device=dev)
        self.kvq = kvq
        # cache read once + the new token's K/V in and its codes out + q in + out
        row = 32 * self.bits + 16  # code bytes + 8 fp16 scales per row
        self.kernel_bytes = B * H * T * 2 * row + 2 * B * H * (512 + row) + B * Hq * 256 * (2 + 4)
        self.step_bytes = self.kernel_bytes
        self.h2d = ["new_k", "new_v", "q"]
        self.d2h = [self.out]
        self.config = {"workload": "long_decode" if self.bits == 4 else "long_decode_q8",
                       "batch": B, "n_q_heads": Hq, "n_kv_heads": H, "head_dim": 256, "ctx": T,
                       "cache": "Q4_0" if self.bits == 4 else "Q8_0",
                       "step": "kvq_decode_step: append 1 token + decode (one call)",
                       "l2": f"{copies} cache copies ({copies * B * H * T * 2 * row / 1e6:.0f} MB) "
                             "rotated per step, inputs > L2"}

    def kernel_call(self, i):
        self.kvq.decode_step(self.caches[i % len(self.caches)], self.new_k, self.new_v, self.q,
                             self.pos, self.T, 1.0 / 16.0, out=self.out, workspace=self.ws)

    def extra(self, call_ms):
        th = self.B * self.H * self.T / call_ms * 1e3
        return {"tok_head_per_s": th, "tok_qhead_per_s": th * self.Hq / self.H}


class LongDecodeQ8(LongDecode):
    """The long-context decode step over a Q8_0 cache (the 8-bit variant):
    544 bytes per token and kv head instead of 288."""
    bits = 8
    kernel_name = "kvq_decode_step (q8_decode_mma_kernel with append + q4_decode_combine_kernel)"
    traffic_key = "q8_decode_long"


class QuantizePrefill(Workload):
    """Quantize-on-append: 4096-token prefill of 8 sequences x 8 kv heads."""
    launches_per_step = 1
    kernel_name = "kvq_quantize_append (q4_append_kernel)"
    traffic_key = "q4_append_prefill"

    def __init__(self, dev):
        import torch
        from hadamard_rotated_bit_fwht_b200 import kvq
        W = synth.WORKLOADS["quantize"]
        B, H, P, A, cap = W["batch"], W["n_kv_heads"], W["prefill"], W["appends"], W["capacity"]
        self.B, self.H, self.P, self.A = B, H, P, A
        k, v = synth.kv_tokens(W["seed"], B, P + A, H, 256, W["outlier_frac"],
                               W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        del k, v
        self.k = bf16_tensor(kb[:, :P], dev)
        self.v = bf16_tensor(vb[:, :P], dev)
        self.singles = [(bf16_tensor(kb[:, P + i:P + i + 1], dev),
                         bf16_tensor(vb[:, P + i:P + i + 1], dev),
                         torch.full((B,), P + i, dtype=torch.int32, device=dev))
                        for i in range(A)]
        self.cache = kvq.Q4Cache.contiguous(B, H, cap, device=dev)
        self.zero = torch.zeros(B, dtype=torch.int32, device=dev)
        self.kvq = kvq
        self.kernel_bytes = self.step_bytes = 2 * B * P * H * (512 + 144)
        self.h2d = ["k", "v"]
        self.d2h = [self.cache.k_scales[:1]]
        self.config = {"workload": "quantize", "batch": B, "n_kv_heads": H, "head_dim": 256,
                       "prefill": P, "dtype_in": "bf16",
                       "step": "kvq_quantize_append(4096-token prefill)",
                       "l2": "inputs 268 MB > L2"}

    def kernel_call(self, i):
        self.kvq.quantize_append(self.cache, self.k, self.v, self.zero)

    def extra(self, call_ms):
        return {"Mtok_s": self.B * self.P / call_ms / 1e3,
                "tok_head_s": self.B * self.P * self.H / call_ms * 1e3}

    def single_token_appends(self):
        """The 256 single-token appends, eager and captured in one CUDA graph."""
        import torch
        s = torch.cuda.current_stream()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for kk, vv, pp in self.singles[:8]:
            self.kvq.quantize_append(self.cache, kk, vv, pp)
        torch.cuda.synchronize()
        a.record(s)
        for kk, vv, pp in self.singles:
            self.kvq.quantize_append(self.cache, kk, vv, pp)
        b.record(s)
        torch.cuda.synchronize()
        eager = a.elapsed_time(b) * 1e3 / self.A
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for kk, vv, pp in self.singles:
                self.kvq.quantize_append(self.cache, kk, vv, pp)
        g.replay()
        torch.cuda.synchronize()
        a.record(s)
        g.replay()
        b.record(s)
        torch.cuda.synchronize()
        graph = a.elapsed_time(b) * 1e3 / self.A
        del g
        return {"us_per_append_eager": eager, "us_per_append_cuda_graph": graph,
                "appends": self.A, "shape": f"batch {self.B}, {self.H} kv heads, 1 token each"}


class PagedDecode(Workload):
    """Batched paged decode: 32 sequences, lengths U[8192, 32768], 256-token
    shuffled pages; a step appends one token per sequence and decodes."""
    launches_per_step = 3
    kernel_name = "kvq_decode_attn, paged (q4_decode_mma_kernel + combine)"
    traffic_key = "q4_decode_paged"

    def __init__(self, dev):
        import torch
        from hadamard_rotated_bit_fwht_b200 import kvq
        W = synth.WORKLOADS["paged_decode"]
        B, H, Hq, ps = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["page_size"]
        self.B, self.H, self.Hq = B, H, Hq
        lens = synth.seq_lens(W["seed"], B, W["ctx_lo"], W["ctx_hi"])
        npp = (lens + ps - 1) // ps
        bt, n_pages = synth.page_table(W["seed"], B, npp, int(npp.max()))
        self.cache = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), device=dev)
        new_k, new_v = [], []
        for b0 in range(0, B, 8):  # generate 8 sequences at a time, append each alone
            Lc = int(lens[b0:b0 + 8].max())
            k, v = synth.kv_tokens(W["seed"] * 100 + b0, 8, Lc, H, 256, W["outlier_frac"],
                                   W["outlier_factor"])
            kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
            del k, v
            for j in range(8):
                L = int(lens[b0 + j])
                one = self.cache.with_block_table(torch.from_numpy(bt[b0 + j:b0 + j + 1]))
                kvq.quantize_append(one, bf16_tensor(kb[j:j + 1, :L], dev),
                                    bf16_tensor(vb[j:j + 1, :L], dev),
                                    torch.zeros(1, dtype=torch.int32, device=dev))
                new_k.append(kb[j, L - 1:L])
                new_v.append(vb[j, L - 1:L])
            del kb, vb
        self.new_k = bf16_tensor(np.stack(new_k), dev)  # (B, 1, H, 256)
        self.new_v = bf16_tensor(np.stack(new_v), dev)
        self.pos = torch.from_numpy(lens - 1).to(dev)
        self.lens = torch.from_numpy(lens).to(dev)
        self.Tm = int(lens.max())
        self.q = bf16_tensor(synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256)), dev)
        self.out = torch.empty((B, Hq, 256), dtype=torch.float32, device=dev)
        self.ws = torch.empty(kvq.decode_attn_workspace(self.cache, B, Hq, self.Tm),
                              dtype=torch.uint8, device=dev)
        self.kvq = kvq
        self.total = int(lens.sum())
        self.kernel_bytes = self.total * H * 288 + B * Hq * 256 * 6
        self.step_bytes = self.kernel_bytes + 2 * B * H * (512 + 144)
        self.h2d = ["new_k", "new_v", "q"]
        self.d2h = [self.out]
        self.config = {"workload": "paged_decode", "batch": B, "n_q_heads": Hq,
                       "n_kv_heads": H, "head_dim": 256, "tokens": self.total,
                       "page_size": ps, "step": "kvq_quantize_append(1 token/seq) + "
                       "kvq_decode_attn", "l2": "cache 369 MB > L2"}

    def pre(self, i):
        self.kvq.quantize_append(self.cache, self.new_k, self.new_v, self.pos)

    def kernel_call(self, i):
        self.kvq.decode_attn(self.cache, self.q, self.lens, self.Tm, 1 / 16, out=self.out,
                             workspace=self.ws)

    def extra(self, call_ms):
        return {"tok_head_per_s": self.total * self.H / call_ms * 1e3}


class OctaveDecode(Workload):
    """Octave k3v4 (head 128, rope 64), 16 requests x 16384 tokens, 32 q / 8 kv
    heads, 256-token shuffled blocks; a step quantizes one new token per
    request into its slot and decodes."""
    launches_per_step = 3  # quantize + split + combine
    kernel_name = "kvq_octave_decode_attn (octave split + combine)"
    traffic_key = "octave_decode"

    def __init__(self, dev):
        import torch
        from hadamard_rotated_bit_fwht_b200 import kvq
        W = synth.WORKLOADS["octave"]
        B, H, Hq, ctx, bs = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["ctx"], W["block_size"]
        self.B, self.H, self.Hq, self.ctx = B, H, Hq, ctx
        self.F = kvq.OctaveFormat(W["head_size"], W["rope_dim"], W["v_bits"])
        self.signs = kvq.sign_words(synth.sign_pattern(128))
        bt, _ = synth.page_table(W["seed"], B, np.full(B, ctx // bs), ctx // bs)
        self.cache = torch.zeros((B * ctx // bs, H, bs, 128), dtype=torch.uint8, device=dev)
        new_k, new_v = [], []
        for r in range(B):
            k, v = synth.kv_tokens(W["seed"] * 100 + r, 1, ctx, H, 128, W["outlier_frac"],
                                   W["outlier_factor"])
            kb, vb = synth.to_bf16_bits(k[0]), synth.to_bf16_bits(v[0])
            slot = torch.from_numpy((bt[r, np.arange(ctx) // bs] * bs + np.arange(ctx) % bs)
                                    .astype(np.int64)).to(dev)
            kd, vd = bf16_tensor(kb, dev), bf16_tensor(vb, dev)
            kvq.octave_quantize(self.F, kd, vd, slot, self.cache, self.signs)
            if r == 0:  # kept for the quantize-throughput figure
                self.qk, self.qv, self.qslot = kd, vd, slot
            new_k.append(kb[ctx - 1])
            new_v.append(vb[ctx - 1])
        self.new_k = bf16_tensor(np.stack(new_k), dev)  # (B, H, 128): token r -> request r
        self.new_v = bf16_tensor(np.stack(new_v), dev)
        self.new_slot = torch.from_numpy((bt[:, (ctx - 1) // bs] * bs + (ctx - 1) % bs)
                                         .astype(np.int64)).to(dev)
        self.q = bf16_tensor(synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 128)), dev)
        self.bt = torch.from_numpy(bt).to(dev)
        self.q2r = torch.arange(B, dtype=torch.int32, device=dev)
        self.q2l = torch.full((B,), ctx, dtype=torch.int32, device=dev)
        self.out = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
        self.ws = torch.empty(kvq.octave_decode_attn_workspace(self.F, B, Hq, ctx),
                              dtype=torch.uint8, device=dev)
        self.kvq = kvq
        self.kernel_bytes = B * ctx * H * 128 + B * Hq * 128 * 6
        self.step_bytes = self.kernel_bytes + B * H * (2 * 256 + 128)
        self.quant_bytes = ctx * H * (2 * 256 + 128)
        self.h2d = ["new_k", "new_v", "q"]
        self.d2h = [self.out]
        self.config = {"workload": "octave", "format": "k3v4", "head_size": 128, "rope_dim": 64,
                       "batch": B, "n_q_heads": Hq, "n_kv_heads": H, "ctx": ctx,
                       "block_size": bs, "step": "kvq_octave_quantize(1 token/request) + "
                       "kvq_octave_decode_attn", "l2": "cache 268 MB > L2"}

    def pre(self, i):
        self.kvq.octave_quantize(self.F, self.new_k, self.new_v, self.new_slot, self.cache,
                                 self.signs)

    def kernel_call(self, i):
        self.kvq.octave_decode_attn(self.F, self.q, self.cache, self.bt, self.q2r, self.q2l,
                                    self.ctx, 128 ** -0.5, self.signs, out=self.out,
                                    workspace=self.ws)

    def quantize_call(self):
        self.kvq.octave_quantize(self.F, self.qk, self.qv, self.qslot, self.cache, self.signs)

    def extra(self, call_ms):
        return {"tok_head_per_s": self.B * self.ctx * self.H / call_ms * 1e3}


WORKLOAD_CLASSES = {"long_decode": LongDecode, "long_decode_q8": LongDecodeQ8,
                    "quantize": QuantizePrefill,
                    "paged_decode": PagedDecode, "octave": OctaveDecode}


# ----------------------------------------------------------------- timing
def capture_graphs(wl, fn):
    """One CUDA graph of fn(i) per distinct step (i mod wl.cycle: the steps of
    a workload rotate through wl.cycle cache copies), captured on a side stream
    after one eager run of each."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graphs = []
    with torch.cuda.stream(s):
        for i in range(wl.cycle):
            fn(i)
        s.synchronize()
        for i in range(wl.cycle):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=s):
                fn(i)
            graphs.append(g)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return graphs


def time_steps(wl, steps, warmup, dist=None):
    """Device time of `steps` steps and the mean device time of the dominant
    call.  Steps replay CUDA graphs of pre(i) + kernel_call(i) back to back
    (the way a decode loop is driven), with CUDA events on the launching stream
    around the whole region only and barrier + synchronize on both sides.  The
    call time comes from a second pass that replays graphs of kernel_call(i)
    alone with events around each replay."""
    import torch
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    step_g = capture_graphs(wl, wl.step)
    call_g = capture_graphs(wl, wl.kernel_call)
    n = wl.cycle
    for i in range(warmup):
        step_g[i % n].replay()
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for i in range(steps):
        step_g[i % n].replay()
    t1.record(s)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for i in range(steps):
        ev[i][0].record(s)
        call_g[i % n].replay()
        ev[i][1].record(s)
    torch.cuda.synchronize()
    call_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    del step_g, call_g
    return total_ms, call_ms


def time_e2e(wl, steps, warmup):
    """The same step with its inputs copied host -> device from pinned memory
    and its output copied back, inside the timed region.  The step's inputs
    (the attributes named in wl.h2d) are moved into one device staging buffer
    so that one copy per step brings all of them."""
    import torch
    dev = getattr(wl, wl.h2d[0]).device
    sizes = [getattr(wl, n).numel() * getattr(wl, n).element_size() for n in wl.h2d]
    offs = [sum((s + 255) // 256 * 256 for s in sizes[:i]) for i in range(len(sizes))]
    total = offs[-1] + (sizes[-1] + 255) // 256 * 256
    stage_d = torch.empty(total, dtype=torch.uint8, device=dev)
    stage_h = torch.empty(total, dtype=torch.uint8).pin_memory()
    for name, off, size in zip(wl.h2d, offs, sizes):
        t = getattr(wl, name)
        view = stage_d[off:off + size].view(t.dtype).view(t.shape)
        view.copy_(t)
        stage_h[off:off + size].copy_(view.view(torch.uint8).reshape(-1).cpu())
        setattr(wl, name, view)
    hout = [torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in wl.d2h]

    def one(i):
        stage_d.copy_(stage_h, non_blocking=True)
        wl.step(i)
        for d, h in zip(wl.d2h, hout):
            h.copy_(d, non_blocking=True)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for i in range(steps):
        one(i)
    b.record(s)
    torch.cuda.synchronize()
    h2d = sum(sizes)
    d2h = sum(t.numel() * t.element_size() for t in hout)
    return a.elapsed_time(b) / steps, h2d, d2h


def time_call(fn, reps, flush=None):
    """Mean device time (ms) of fn() over reps; an L2 flush runs before each rep
    outside the timed events."""
    import torch
    s = torch.cuda.current_stream()
    ts = []
    for _ in range(reps):
        if flush is not None:
            flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(s)
        fn()
        b.record(s)
        ts.append((a, b))
    torch.cuda.synchronize()
    return float(np.mean([a.elapsed_time(b) for a, b in ts]))


def other_workloads(dev, main_name, reps, peak):
    """Per-call timing of every workload other than the main one."""
    import torch
    flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.fill_(1)

    res = {}
    for name, cls in WORKLOAD_CLASSES.items():
        if name == main_name:
            continue
        wl = cls(dev)
        for i in range(3):
            wl.kernel_call(i)
        ms = time_call(lambda: wl.kernel_call(0), reps, flush)
        gbs = wl.kernel_bytes / ms / 1e6
        res[name] = {"call": wl.kernel_name, "ms": ms, "GB_s": gbs, "frac_of_peak": gbs / peak,
                     "bytes": wl.kernel_bytes, "config": wl.config, **wl.extra(ms)}
        if isinstance(wl, QuantizePrefill):
            res["quantize_single_token_append"] = wl.single_token_appends()
        if isinstance(wl, OctaveDecode):
            for _ in range(2):
                wl.quantize_call()
            qms = time_call(wl.quantize_call, reps, flush)
            res["octave_quantize"] = {
                "ms": qms, "GB_s": wl.quant_bytes / qms / 1e6,
                "frac_of_peak": wl.quant_bytes / qms / 1e6 / peak, "Mtok_s": wl.ctx / qms / 1e3,
                "shape": f"{wl.ctx} tokens x {wl.H} kv heads, bf16 -> 128-byte slots"}
        del wl
        torch.cuda.synchronize()
    del flush_buf
    return res


# ----------------------------------------------------------------- CPU oracle leg
def cpu_oracle_long_decode(steps: int, warmup: int = 0, threads: int = 1):
    """Time the oracle on the long-context decode step on the host.  With one
    thread the sample is kv head 0 (its 8 query heads over all 131072 tokens,
    1/4 of a step); with more, the whole step (all 4 kv heads, one
    (sequence, kv head) unit per thread).  The cache is built once (untimed);
    each step appends the new token and decodes (`warmup` untimed steps
    first).  Returns (GB/s, seconds, sample, threads used)."""
    import oracle
    W = synth.WORKLOADS["long_decode"]
    T, Hq, H = W["ctx"], W["n_q_heads"], W["n_kv_heads"]
    G = Hq // H
    nh = 1 if threads <= 1 else H
    k, v = synth.kv_tokens(W["seed"], 1, T, H, 256, W["outlier_frac"], W["outlier_factor"])
    kb = np.ascontiguousarray(synth.to_bf16_bits(k)[:, :, :nh])
    vb = np.ascontiguousarray(synth.to_bf16_bits(v)[:, :, :nh])
    del k, v
    q = synth.to_bf16_bits(synth.queries(W["seed"], 1, Hq, 256))[:, :G * nh].copy()
    oc = oracle.Q4Cache(T * nh, nh, max_tokens=T)
    oc.append(kb, vb, [0], threads=threads)
    used = min(threads, nh)

    def step():
        oc.append(kb[:, T - 1:T], vb[:, T - 1:T], [T - 1])
        oc.decode_attn(q, [T], 1 / 16, threads=threads)

    for _ in range(warmup):
        step()
    t = time.perf_counter()
    for _ in range(steps):
        step()
    dt = time.perf_counter() - t
    bytes_per_step = nh * (T * 288 + G * 256 * 6 + 2 * (512 + 144))
    if nh == 1:
        sample = (f"{steps} steps of the long-context decode step restricted to kv head 0 "
                  f"(its {G} query heads, {T} tokens): 1/{H} of a GPU step, 1 thread")
    else:
        sample = (f"{steps} whole long-context decode steps ({H} kv heads x {G} query heads, "
                  f"{T} tokens), one (sequence, kv head) unit per thread")
    return bytes_per_step * steps / dt / 1e9, dt, sample, used


def cpu_oracle_quantize(threads: int):
    """Oracle quantize-on-append of the whole 4096-token prefill (8 sequences x
    8 kv heads), (sequence, 512-token chunk) units on threads."""
    import oracle
    W = synth.WORKLOADS["quantize"]
    B, H, P = W["batch"], W["n_kv_heads"], W["prefill"]
    k, v = synth.kv_tokens(W["seed"], B, P, H, 256, W["outlier_frac"], W["outlier_factor"])
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    del k, v
    oc = oracle.Q4Cache(B * H * W["capacity"], H, max_tokens=W["capacity"])
    t = time.perf_counter()
    oc.append(kb, vb, np.zeros(B, np.int32), threads=threads)
    dt = time.perf_counter() - t
    return {"value": B * P / dt / 1e6, "unit": "Mtok/s", "seconds": dt,
            "GB_s": 2 * B * P * H * (512 + 144) / dt / 1e9,
            "cores": min(threads, B * (P // 512)), "kind": "oracle",
            "sample": f"the whole prefill ({B} sequences x {P} tokens x {H} kv heads)"}


def cpu_oracle_paged(threads: int):
    """Oracle decode of the first 8 of the 32 paged sequences (the benchmark's
    first generation group; 16 (sequence, kv head) units on threads)."""
    import oracle
    W = synth.WORKLOADS["paged_decode"]
    B, H, Hq, ps = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["page_size"]
    n = 8
    lens = synth.seq_lens(W["seed"], B, W["ctx_lo"], W["ctx_hi"])[:n]
    npp = (lens + ps - 1) // ps
    bt, n_pages = synth.page_table(W["seed"], n, npp, int(npp.max()))
    k, v = synth.kv_tokens(W["seed"] * 100, n, int(lens.max()), H, 256, W["outlier_frac"],
                           W["outlier_factor"])
    kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
    del k, v
    oc = oracle.Q4Cache(n_pages * H * ps, H, block_table=bt, page_size=ps)
    for b in range(n):
        oc.with_block_table(bt[b:b + 1]).append(kb[b:b + 1, :lens[b]], vb[b:b + 1, :lens[b]],
                                                np.zeros(1, np.int32), threads=threads)
    q = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256))[:n]
    reps = 4
    t = time.perf_counter()
    for _ in range(reps):
        oc.decode_attn(q, lens, 1 / 16, threads=threads)
    dt = time.perf_counter() - t
    return {"value": reps * int(lens.sum()) * H * 288 / dt / 1e9, "unit": "GB/s", "seconds": dt,
            "cores": min(threads, n * H), "kind": "oracle",
            "sample": f"{reps} decodes of {n} of the {B} sequences ({int(lens.sum())} tokens, "
                      f"{H} kv heads)"}


def cpu_oracle_octave(threads: int):
    """Oracle Octave k3v4 decode of 4 of the 16 requests (16384 tokens each,
    all 32 query heads; one query token per thread)."""
    import oracle
    W = synth.WORKLOADS["octave"]
    H, Hq, ctx, bs = W["n_kv_heads"], W["n_q_heads"], W["ctx"], W["block_size"]
    n = 4
    fmt = (W["head_size"], W["rope_dim"], W["v_bits"], 0)
    signs = synth.sign_pattern(128)
    cache = np.zeros((n * ctx // bs, H, bs, 128), np.uint8)
    bt = np.arange(n * ctx // bs, dtype=np.int32).reshape(n, ctx // bs)
    for r in range(n):
        k, v = synth.kv_tokens(W["seed"] * 100 + r, 1, ctx, H, 128, W["outlier_frac"],
                               W["outlier_factor"])
        slots = oracle.octave_quantize(synth.to_bf16_bits(k[0]), synth.to_bf16_bits(v[0]), fmt,
                                       signs, threads=threads)
        del k, v
        cache[r * ctx // bs:(r + 1) * ctx // bs] = slots.reshape(ctx // bs, bs, H, 128).transpose(0, 2, 1, 3)
    q = synth.to_bf16_bits(synth.queries(W["seed"], W["batch"], Hq, 128))[:n]
    t = time.perf_counter()
    oracle.octave_attention(q, cache, bt, np.arange(n, dtype=np.int32), np.full(n, ctx, np.int32),
                            fmt, 128 ** -0.5, signs, threads=threads)
    dt = time.perf_counter() - t
    return {"value": n * ctx * H * 128 / dt / 1e9, "unit": "GB/s", "seconds": dt,
            "cores": min(threads, n), "kind": "oracle",
            "sample": f"decode of {n} of the {W['batch']} requests ({ctx} tokens, {Hq} q heads)"}


def cpu_baselines(threads: int):
    """The headline (long-context decode) oracle figure on all cores and on one,
    plus bounded multi-core samples of the other workloads."""
    # about 3 s of wall time each: 8 quarter steps on one core, 6 whole steps
    # (about 12 s of CPU work on 4 threads)
    gbs1, dt1, sample1, _ = cpu_oracle_long_decode(steps=8, threads=1)
    gbs, dt, sample, used = cpu_oracle_long_decode(steps=6, threads=threads)
    per = {"long_decode": {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle",
                           "sample": sample, "seconds": dt},
           "long_decode_1_core": {"value": gbs1, "unit": "GB/s", "cores": 1, "kind": "oracle",
                                  "sample": sample1, "seconds": dt1},
           "quantize": cpu_oracle_quantize(threads),
           "paged_decode": cpu_oracle_paged(threads),
           "octave": cpu_oracle_octave(threads)}
    return {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle", "sample": sample,
            "seconds": dt, "host_threads": threads, "single_core": per["long_decode_1_core"],
            "workloads": per}


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    import oracle
    threads = oracle.host_threads()
    # bounded sample: at most 8 timed and 2 warm-up whole oracle steps (about
    # 0.5 s of wall time and 2 s of CPU work each on 4 threads)
    steps = max(1, min(args.steps, 8))
    warm = max(0, min(args.warmup, 2))
    gbs, dt, sample, used = cpu_oracle_long_decode(steps, warm, threads=threads)
    W = synth.WORKLOADS["long_decode"]
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": warm, "ms_per_step": dt * 1e3 / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "long_decode", "batch": W["batch"], "n_q_heads": W["n_q_heads"],
                   "n_kv_heads": W["n_kv_heads"], "head_dim": 256, "ctx": W["ctx"],
                   "cache": "Q4_0",
                   "step": "kvq_decode_step: append 1 token + decode (one call)",
                   "parallelism": f"replicas x{args.gpus}"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": used, "kind": "oracle",
                         "sample": sample, "host_threads": threads},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ----------------------------------------------------------------- main
def busy(wl, seconds, start):
    """Keep the GPU on the step for a while (for the clock sampler)."""
    import torch
    t_end = time.time() + seconds
    i = start
    while time.time() < t_end:
        wl.step(i)
        i += 1
        if i % 64 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    return i


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--workload", default="long_decode", choices=list(WORKLOAD_CLASSES))
    ap.add_argument("--no-workloads", action="store_true",
                    help="report the main workload only")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as tdist
        torch.cuda.set_device(local)
        tdist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
        dist = tdist
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    from hadamard_rotated_bit_fwht_b200 import build as kbuild
    if rank == 0:
        kbuild.build()
    if dist is not None:
        dist.barrier()
    peak, peak_kind = load_peaks()

    wl = WORKLOAD_CLASSES[args.workload](dev)
    clocks = ClockSampler(local)
    clocks.start()
    i = busy(wl, 0.5, 0)
    total_ms, call_ms = time_steps(wl, args.steps, args.warmup, dist)
    busy(wl, 0.5, i)
    clk = clocks.stop()

    ms_step, call_ms = max_over_ranks([total_ms / args.steps, call_ms], dist, dev)
    value = job_throughput_gbs(wl.step_bytes, world, ms_step)
    achieved = wl.kernel_bytes / call_ms / 1e6
    e2e_ms, h2d, d2h = time_e2e(wl, max(20, args.steps // 10), 5)
    (e2e_ms,) = max_over_ranks([e2e_ms], dist, dev)
    e2e_value = job_throughput_gbs(wl.step_bytes, world, e2e_ms)
    info = {"config": wl.config, "extra": wl.extra(call_ms), "kernel": wl.kernel_name,
            "kernel_bytes": wl.kernel_bytes, "traffic_key": wl.traffic_key,
            "launches": wl.launches_per_step}
    del wl
    torch.cuda.synchronize()

    workloads = None
    if not args.no_workloads and rank == 0:
        workloads = other_workloads(dev, args.workload, reps=20, peak=peak)
    if dist is not None:
        dist.barrier()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == "long_decode":
        import oracle
        cpu = cpu_baselines(oracle.host_threads())

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {**info["config"], "parallelism": f"replicas x{world}",
                       "timing": "steps replay CUDA graphs back to back (one per input copy); "
                                 "e2e runs the public API eagerly"},
            "frac_of_peak": value / world / peak,
            **info["extra"],
            "roofline": {"bound": "hbm", "kernel": info["kernel"], "achieved": achieved,
                         "peak": peak, "peak_kind": peak_kind, "unit": "GB/s",
                         "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": info["kernel_bytes"],
                         "traffic": recorded_traffic(info["traffic_key"])},
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": info["launches"] * args.steps,
            "clocks": clk,
            "cpu_baseline": cpu,
            "workloads": workloads,
            "hbm_nominal_gbs": HBM_NOMINAL,
        }
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
