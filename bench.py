"""Benchmark of the Hadamard-rotated Q4_0 KV cache on B200.

One step = one pass of the whole hot path on the long-context decode workload
(1 sequence, 131072 tokens, 32 query / 4 kv heads, D = 256, bf16 inputs):
kvq_quantize_append of the new token's K and V (rotate + Q4_0 + store), then
kvq_decode_attn over the whole cache (rotate q, stream and dequantize the
nibbles, online softmax, split-K combine, back-rotation).

`value` is decode-step HBM throughput in GB/s: algorithmic bytes per step
(every cache byte read once, inputs read and outputs written once) / device
time per step, summed over ranks.  Three copies of the cache (453 MB, over 3x
the 126 MB L2) are rotated so no step reads bytes the previous step left in L2.
The other workloads (quantize prefill, paged decode, Octave) are timed the same
way and reported under "workloads".

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl kvq|reference]
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


def kernel_source_hash():
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "hadamard_rotated_bit_fwht_b200", "csrc")
    for f in sorted(os.listdir(csrc)):
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str):
    """DRAM bytes per launch from a committed ncu capture, only if the kernel
    sources are unchanged since it was taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash():
        return None
    return e.get("bytes_per_launch")


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
    return torch.from_numpy(a).view(torch.bfloat16).to(dev)


class LongDecode:
    """Long-context decode workload and its per-step byte count."""

    def __init__(self, dev, copies=3):
        import torch
        from hadamard_rotated_bit_fwht_b200 import kvq
        W = synth.WORKLOADS["long_decode"]
        self.W = W
        B, H, T, Hq = W["batch"], W["n_kv_heads"], W["ctx"], W["n_q_heads"]
        self.B, self.H, self.T, self.Hq = B, H, T, Hq
        k, v = synth.kv_tokens(W["seed"], B, T, H, 256, W["outlier_frac"], W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        del k, v
        self.host_k, self.host_v = kb, vb
        kd, vd = bf16_tensor(kb, dev), bf16_tensor(vb, dev)
        self.caches = []
        zero = torch.zeros(B, dtype=torch.int32, device=dev)
        for _ in range(copies):
            c = kvq.Q4Cache.contiguous(B, H, T, device=dev)
            kvq.quantize_append(c, kd, vd, zero)
            self.caches.append(c)
        del kd, vd
        self.q_host = synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256))
        self.q = bf16_tensor(self.q_host, dev)
        # the step's new token: the last position of each sequence
        self.new_k_host = np.ascontiguousarray(kb[:, T - 1:T])
        self.new_v_host = np.ascontiguousarray(vb[:, T - 1:T])
        self.new_k = bf16_tensor(self.new_k_host, dev)
        self.new_v = bf16_tensor(self.new_v_host, dev)
        self.pos = torch.full((B,), T - 1, dtype=torch.int32, device=dev)
        self.lens = torch.full((B,), T, dtype=torch.int32, device=dev)
        self.out = torch.empty((B, Hq, 256), dtype=torch.float32, device=dev)
        ws = kvq.decode_attn_workspace(self.caches[0], B, Hq, T)
        self.ws = torch.empty(ws, dtype=torch.uint8, device=dev)
        self.kvq = kvq
        torch.cuda.synchronize()

    def decode_bytes(self):
        return (self.B * self.H * self.T * 288 + self.B * self.Hq * 256 * 2
                + self.B * self.Hq * 256 * 4)

    def append_bytes(self):
        return 2 * self.B * self.H * (512 + 144)

    def step_bytes(self):
        return self.decode_bytes() + self.append_bytes()

    def append(self, i):
        self.kvq.quantize_append(self.caches[i % len(self.caches)], self.new_k, self.new_v, self.pos)

    def decode(self, i):
        self.kvq.decode_attn(self.caches[i % len(self.caches)], self.q, self.lens, self.T,
                             1.0 / 16.0, out=self.out, workspace=self.ws)

    def step(self, i):
        self.append(i)
        self.decode(i)

    launches_per_step = 3  # append + decode split + combine


def time_steps(wl, steps, warmup, dist=None):
    """Device time of `steps` steps (CUDA events around the region, barrier and
    synchronize on both sides); also per-launch time of the decode call."""
    import torch
    for i in range(warmup):
        wl.step(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(s)
    for i in range(steps):
        wl.append(i)
        ev[i][0].record(s)
        wl.decode(i)
        ev[i][1].record(s)
    t1.record(s)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    total_ms = t0.elapsed_time(t1)
    dec_ms = float(np.mean([a.elapsed_time(b) for a, b in ev]))
    return total_ms, dec_ms


def time_e2e(wl, steps, warmup):
    """Same step through the C ABI with host buffers: H2D of the new token's
    K, V and the query from pinned memory, the step, D2H of the output."""
    import torch
    dev = wl.q.device
    hk = torch.from_numpy(wl.new_k_host).view(torch.bfloat16).pin_memory()
    hv = torch.from_numpy(wl.new_v_host).view(torch.bfloat16).pin_memory()
    hq = torch.from_numpy(wl.q_host).view(torch.bfloat16).pin_memory()
    ho = torch.empty(wl.out.shape, dtype=torch.float32).pin_memory()

    def one(i):
        wl.new_k.copy_(hk, non_blocking=True)
        wl.new_v.copy_(hv, non_blocking=True)
        wl.q.copy_(hq, non_blocking=True)
        wl.step(i)
        ho.copy_(wl.out, non_blocking=True)

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
    h2d = hk.numel() * 2 + hv.numel() * 2 + hq.numel() * 2
    d2h = ho.numel() * 4
    _ = dev
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


def other_workloads(dev, reps, peak):
    """Quantize prefill / single-token appends, paged decode and Octave."""
    import torch
    from hadamard_rotated_bit_fwht_b200 import kvq
    flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device=dev)

    def flush():
        flush_buf.fill_(1)

    res = {}
    # ---- quantize-on-append (B=8, Hkv=8, 4096-token prefill, 256 appends)
    W = synth.WORKLOADS["quantize"]
    B, H, P, A, cap = W["batch"], W["n_kv_heads"], W["prefill"], W["appends"], W["capacity"]
    k, v = synth.kv_tokens(W["seed"], B, P + A, H, 256, W["outlier_frac"], W["outlier_factor"])
    kd, vd = bf16_tensor(synth.to_bf16_bits(k), dev), bf16_tensor(synth.to_bf16_bits(v), dev)
    del k, v
    cache = kvq.Q4Cache.contiguous(B, H, cap, device=dev)
    kp, vp = kd[:, :P].contiguous(), vd[:, :P].contiguous()
    zero = torch.zeros(B, dtype=torch.int32, device=dev)
    for _ in range(3):
        kvq.quantize_append(cache, kp, vp, zero)
    ms = time_call(lambda: kvq.quantize_append(cache, kp, vp, zero), reps, flush)
    nbytes = 2 * B * P * H * (512 + 144)
    res["quantize_prefill"] = {
        "ms": ms, "GB_s": nbytes / ms / 1e6, "frac_of_peak": nbytes / ms / 1e6 / peak,
        "Mtok_s": B * P / ms / 1e3, "tok_head_s": B * P * H / ms * 1e3, "bytes": nbytes,
        "shape": f"batch {B}, {H} kv heads, {P}-token prefill, bf16 -> Q4_0"}
    singles = [(kd[:, P + i:P + i + 1].contiguous(), vd[:, P + i:P + i + 1].contiguous(),
                torch.full((B,), P + i, dtype=torch.int32, device=dev)) for i in range(A)]
    torch.cuda.synchronize()
    s = torch.cuda.current_stream()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s)
    for kk, vv, pp in singles:
        kvq.quantize_append(cache, kk, vv, pp)
    b.record(s)
    torch.cuda.synchronize()
    us_eager = a.elapsed_time(b) * 1e3 / A
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for kk, vv, pp in singles:
            kvq.quantize_append(cache, kk, vv, pp)
    g.replay()
    torch.cuda.synchronize()
    a.record(s)
    g.replay()
    b.record(s)
    torch.cuda.synchronize()
    res["quantize_single_token_append"] = {
        "us_per_append_eager": us_eager, "us_per_append_cuda_graph": a.elapsed_time(b) * 1e3 / A,
        "appends": A, "shape": f"batch {B}, {H} kv heads, 1 token each"}
    del g, singles, kd, vd, kp, vp, cache

    # ---- paged decode (B=32, 16 q / 2 kv heads, lens U[8192, 32768], 256-token pages)
    W = synth.WORKLOADS["paged_decode"]
    B, H, Hq, ps = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["page_size"]
    lens = synth.seq_lens(W["seed"], B, W["ctx_lo"], W["ctx_hi"])
    npp = (lens + ps - 1) // ps
    maxp = int(npp.max())
    bt, n_pages = synth.page_table(W["seed"], B, npp, maxp)
    pc = kvq.Q4Cache.paged(n_pages, H, ps, torch.from_numpy(bt), device=dev)
    Tm = int(lens.max())
    for b0 in range(0, B, 8):  # generate 8 sequences at a time, append each alone
        Lc = int(lens[b0:b0 + 8].max())
        k, v = synth.kv_tokens(W["seed"] * 100 + b0, 8, Lc, H, 256, W["outlier_frac"],
                               W["outlier_factor"])
        kb, vb = synth.to_bf16_bits(k), synth.to_bf16_bits(v)
        del k, v
        for j in range(8):
            L = int(lens[b0 + j])
            one = pc.with_block_table(torch.from_numpy(bt[b0 + j:b0 + j + 1]))
            kvq.quantize_append(one, bf16_tensor(np.ascontiguousarray(kb[j:j + 1, :L]), dev),
                                bf16_tensor(np.ascontiguousarray(vb[j:j + 1, :L]), dev),
                                torch.zeros(1, dtype=torch.int32, device=dev))
        del kb, vb
    q = bf16_tensor(synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 256)), dev)
    lens_d = torch.from_numpy(lens).to(dev)
    out = torch.empty((B, Hq, 256), dtype=torch.float32, device=dev)
    wsz = kvq.decode_attn_workspace(pc, B, Hq, Tm)
    ws = torch.empty(wsz, dtype=torch.uint8, device=dev)

    def dec():
        kvq.decode_attn(pc, q, lens_d, Tm, 1 / 16, out=out, workspace=ws)

    for _ in range(3):
        dec()
    ms = time_call(dec, reps, flush)
    tot = int(lens.sum())
    nbytes = tot * H * 288 + B * Hq * 256 * 6
    res["paged_decode"] = {
        "ms": ms, "GB_s": nbytes / ms / 1e6, "frac_of_peak": nbytes / ms / 1e6 / peak,
        "tok_head_s": tot * H / ms * 1e3, "bytes": nbytes,
        "shape": f"batch {B}, {Hq} q / {H} kv heads, {tot} tokens, 256-token shuffled pages"}
    del pc, ws

    # ---- Octave k3v4 (B=16, 32 q / 8 kv heads, head 128, ctx 16384, 256-token blocks)
    W = synth.WORKLOADS["octave"]
    B, H, Hq, ctx, bs = W["batch"], W["n_kv_heads"], W["n_q_heads"], W["ctx"], W["block_size"]
    F = kvq.OctaveFormat(W["head_size"], W["rope_dim"], W["v_bits"])
    signs = kvq.sign_words(synth.sign_pattern(128))
    nb = B * ctx // bs
    bt, _ = synth.page_table(W["seed"], B, np.full(B, ctx // bs), ctx // bs)
    ocache = torch.zeros((nb, H, bs, 128), dtype=torch.uint8, device=dev)
    qtime = []
    for r in range(B):
        k, v = synth.kv_tokens(W["seed"] * 100 + r, 1, ctx, H, 128, W["outlier_frac"],
                               W["outlier_factor"])
        kd = bf16_tensor(synth.to_bf16_bits(k[0]), dev)
        vd = bf16_tensor(synth.to_bf16_bits(v[0]), dev)
        slot = torch.from_numpy((bt[r, np.arange(ctx) // bs] * bs + np.arange(ctx) % bs)
                                .astype(np.int64)).to(dev)
        kvq.octave_quantize(F, kd, vd, slot, ocache, signs)
        if r == 0:
            for _ in range(2):
                kvq.octave_quantize(F, kd, vd, slot, ocache, signs)
            qtime.append(time_call(lambda: kvq.octave_quantize(F, kd, vd, slot, ocache, signs),
                                   reps, flush))
    qo = bf16_tensor(synth.to_bf16_bits(synth.queries(W["seed"], B, Hq, 128)), dev)
    btd = torch.from_numpy(bt).to(dev)
    q2r = torch.arange(B, dtype=torch.int32, device=dev)
    q2l = torch.full((B,), ctx, dtype=torch.int32, device=dev)
    oout = torch.empty((B, Hq, 128), dtype=torch.float32, device=dev)
    wsz = kvq.octave_decode_attn_workspace(F, B, Hq, ctx)
    ows = torch.empty(wsz, dtype=torch.uint8, device=dev)

    def odec():
        kvq.octave_decode_attn(F, qo, ocache, btd, q2r, q2l, ctx, 128 ** -0.5, signs, out=oout,
                               workspace=ows)

    for _ in range(3):
        odec()
    ms = time_call(odec, reps, flush)
    nbytes = B * ctx * H * 128 + B * Hq * 128 * 6
    qbytes = ctx * H * (2 * 128 * 2 + 128)
    res["octave_decode"] = {
        "ms": ms, "GB_s": nbytes / ms / 1e6, "frac_of_peak": nbytes / ms / 1e6 / peak,
        "tok_head_s": B * ctx * H / ms * 1e3, "bytes": nbytes,
        "shape": f"k3v4 head 128 rope 64, batch {B}, {Hq} q / {H} kv heads, ctx {ctx}, "
                 "256-token shuffled blocks"}
    res["octave_quantize"] = {
        "ms": qtime[0], "GB_s": qbytes / qtime[0] / 1e6,
        "frac_of_peak": qbytes / qtime[0] / 1e6 / peak, "Mtok_s": ctx / qtime[0] / 1e3,
        "shape": f"{ctx} tokens x {H} kv heads, bf16 -> 128-byte slots"}
    del ocache, flush_buf
    torch.cuda.synchronize()
    return res


# ----------------------------------------------------------------- CPU oracle leg
def cpu_oracle_long_decode(steps: int):
    """Time the oracle on the same workload on the host: the cache of kv head 0
    (131072 tokens) is built once (untimed), then each step appends the new
    token and decodes its 8 query heads.  Returns (GB/s, seconds, sample)."""
    import oracle
    W = synth.WORKLOADS["long_decode"]
    T, Hq, H = W["ctx"], W["n_q_heads"], W["n_kv_heads"]
    G = Hq // H
    k, v = synth.kv_tokens(W["seed"], 1, T, H, 256, W["outlier_frac"], W["outlier_factor"])
    kb = np.ascontiguousarray(synth.to_bf16_bits(k)[:, :, :1])
    vb = np.ascontiguousarray(synth.to_bf16_bits(v)[:, :, :1])
    del k, v
    q = synth.to_bf16_bits(synth.queries(W["seed"], 1, Hq, 256))[:, :G].copy()
    oc = oracle.Q4Cache(T, 1, max_tokens=T)
    oc.append(kb, vb, [0])
    t = time.perf_counter()
    for _ in range(steps):
        oc.append(kb[:, T - 1:T], vb[:, T - 1:T], [T - 1])
        oc.decode_attn(q, [T], 1 / 16)
    dt = time.perf_counter() - t
    bytes_per_step = T * 288 + G * 256 * 6 + 2 * (512 + 144)
    sample = (f"{steps} steps of the long-context decode step restricted to kv head 0 "
              f"(its {G} query heads, {T} tokens): 1/{H} of a GPU step")
    return bytes_per_step * steps / dt / 1e9, dt, sample


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    steps = max(1, min(args.steps, 8))
    gbs, dt, sample = cpu_oracle_long_decode(steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s",
        "n_gpus": args.gpus, "steps": steps, "warmup": 0, "ms_per_step": dt * 1e3 / steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": "long_decode", "batch": 1, "n_q_heads": 32, "n_kv_heads": 4,
                   "head_dim": 256, "ctx": 131072, "parallelism": "replicas"},
        "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))


# ----------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", default="kvq", choices=["kvq", "reference"])
    ap.add_argument("--no-workloads", action="store_true", help="skip the other workloads")
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
    if rank == 0 or world == 1:
        kbuild.build()
    if dist is not None:
        dist.barrier()
    peak, peak_kind = load_peaks()

    wl = LongDecode(dev)
    clocks = ClockSampler(torch.cuda.current_device() if "CUDA_VISIBLE_DEVICES" not in os.environ
                          else local)
    clocks.start()
    # keep the GPU busy ~0.5 s before and after the timed region for the sampler
    t_end = time.time() + 0.5
    i = 0
    while time.time() < t_end:
        wl.step(i)
        i += 1
        if i % 200 == 0:
            torch.cuda.synchronize()
    total_ms, dec_ms = time_steps(wl, args.steps, args.warmup, dist)
    t_end = time.time() + 0.5
    while time.time() < t_end:
        wl.step(i)
        i += 1
        if i % 200 == 0:
            torch.cuda.synchronize()
    torch.cuda.synchronize()
    clk = clocks.stop()

    ms_step = total_ms / args.steps
    if dist is not None:
        t = torch.tensor([ms_step, dec_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms_step, dec_ms = float(t[0]), float(t[1])
    value = wl.step_bytes() * world / ms_step / 1e6  # GB/s, whole job
    achieved = wl.decode_bytes() / dec_ms / 1e6
    e2e_ms, h2d, d2h = time_e2e(wl, max(50, args.steps // 10), 10)
    if dist is not None:
        t = torch.tensor([e2e_ms], dtype=torch.float64, device=dev)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        e2e_ms = float(t[0])
    e2e_value = wl.step_bytes() * world / e2e_ms / 1e6

    workloads = None
    if not args.no_workloads and rank == 0:
        workloads = other_workloads(dev, reps=20, peak=peak)
    if dist is not None:
        dist.barrier()

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        gbs, dt, sample = cpu_oracle_long_decode(steps=5)
        cpu = {"value": gbs, "unit": "GB/s", "cores": 1, "kind": "oracle", "sample": sample,
               "seconds": dt}

    if rank == 0:
        tok_head = wl.B * wl.H * wl.T / dec_ms * 1e3
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": "long_decode", "batch": wl.B, "n_q_heads": wl.Hq,
                       "n_kv_heads": wl.H, "head_dim": 256, "ctx": wl.T,
                       "step": "kvq_quantize_append(1 token) + kvq_decode_attn",
                       "l2": "3 cache copies (453 MB) rotated per step, inputs > L2",
                       "parallelism": f"replicas x{world}"},
            "frac_of_peak": value / world / peak,
            "tok_head_per_s": tok_head, "tok_qhead_per_s": tok_head * wl.Hq / wl.H,
            "roofline": {"bound": "hbm", "kernel": "kvq_decode_attn (split + combine launches)",
                         "achieved": achieved, "peak": peak, "peak_kind": peak_kind,
                         "unit": "GB/s", "frac": achieved / peak,
                         "algorithmic_bytes_per_launch": wl.decode_bytes(),
                         "traffic": recorded_traffic("q4_decode_long")},
            "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": wl.launches_per_step * args.steps,
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
