#!/usr/bin/env python3
"""Benchmark of the hot path on the throughput workload (the largest of the
five configurations): batch 64, 32 query heads / 8 kv heads, head dim 128,
8192 prefilled tokens + 256 tokens streamed one per decode step, NSN +
plain Hadamard, INT4 codes.

One step = one pass of the whole path over one batch:
  kvq_quantize_block over the 8192-token prefill (K and V), then 256 x
  [kvq_append_token (two of them flush a block) + kvq_decode_attention].
`value` = algorithmic bytes of every call in the step / step time (GB/s);
decode dominates it.  Inputs (1 GiB each of K and V, the queries and the
streamed tokens) are resident in HBM before the timed region; the 604 MB
packed cache is larger than the 126 MB L2, so no flush is needed between
iterations.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]

Under torchrun each rank runs its own batch (weak scaling, no collective on
the data path); the step time is the max over ranks.  `--impl reference`
times the CPU oracle (the plain C reference of the method) on the host
cores over a bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
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

from kv_cache_bit_b200 import accounting, synth  # noqa: E402

WORKLOAD = "throughput"
MODE = "nsn+hadamard"
BITS = 4
# the mode each workload is quoted in (the throughput workload is the default)
WORKLOAD_MODES = {"tiny": "nsep+pchan", "qwen2-7b-gqa": "nsep+pchan", "pythia-6.9b-mha": "nsep+pchan",
                  "llama-long-ctx": "rht+nsep+pchan", "throughput": "nsn+hadamard"}
METRIC = "INT4-KV decode attention GB/s (% of HBM peak) & tokens/s; quantize GB/s"


# The sources the decode kernels are built from (the host file holds their
# launch configuration); the quantizer's own files are not among them.
KERNEL_SOURCES = ["kvq_api.cu", "kvq_decode_mma.cuh", "kvq_decode_simple.cuh", "kvq_device.cuh"]
TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "decode_traffic_throughput.md")


def decode_traffic():
    """DRAM bytes of one decode call from the committed ncu summary, or None
    when the kernels have changed since it was captured."""
    import hashlib
    try:
        text = open(TRAFFIC_PROFILE).read()
        fields = dict(ln.split(":", 1) for ln in text.splitlines() if ln.startswith(("traffic_bytes_per_call:",
                                                                                      "source_sha256:")))
        h = hashlib.sha256()
        for f in KERNEL_SOURCES:
            with open(os.path.join(ROOT, "kv_cache_bit_b200", "csrc", f), "rb") as fh:
                h.update(fh.read())
        if h.hexdigest() != fields["source_sha256"].strip():
            return None
        return float(fields["traffic_bytes_per_call:".rstrip(":")].strip())
    except Exception:
        return None


def measured_peak_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def flags_of(mode: str) -> int:
    names, _ = synth.MODES[mode]
    m = {"NORM_SEP": 1, "PER_CHANNEL": 2, "NSN": 4, "HADAMARD": 8, "DQ": 16}
    f = 0
    for n in names:
        f |= m[n]
    return f


# ------------------------------------------------------------------ clocks

class ClockSampler:
    """nvidia-smi samples of the SM clock and throttle reasons while the
    timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.proc = None
        self.lines = []

    def start(self):
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "200"]
        if self.uuid:
            cmd[1:1] = ["-i", self.uuid]
        try:
            self.proc = subprocess.Popen(cmd, stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except Exception:
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
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------ oracle sample

def run_oracle_sample(w, mode, bits, pairs, threads, decode_seconds, data=None):
    """The CPU oracle over `pairs` (batch row, kv head) slices of the
    workload: quantize of the prefill (K and V), then decode steps over the
    quantized cache (each one dequantize + fp64 attention of the slices'
    query heads with a fresh query) until about `decode_seconds` of decode
    work.  `data` = (K, V) fp16 [pairs, 1, S, d] of those slices (else they
    are drawn here).  Returns (bytes, seconds, decode steps, quantize seconds,
    oracle state): the algorithmic bytes of the quantize and of every decode
    step, with the same accounting as the GPU path, and the oracle's caches
    with the exact products of their codes (for the parity sample)."""
    import oracle
    names, seeded = synth.MODES[mode]
    flags = flags_of(mode)
    cfg = oracle.Cfg(d=w.d, bits=bits, flags=flags,
                     signs=oracle.make_signs(synth.SIGN_SEED, w.d) if seeded else None)
    G = w.Hq // w.Hkv
    ws = w.scaled(B=max(1, (pairs + w.Hkv - 1) // w.Hkv))
    if data is None:
        K, V = synth.kv(ws)
        Kb = K.reshape(-1, 1, w.S, w.d)[:pairs]
        Vb = V.reshape(-1, 1, w.S, w.d)[:pairs]
    else:
        Kb, Vb = data
    k16 = np.ascontiguousarray(Kb).view(np.uint16)
    v16 = np.ascontiguousarray(Vb).view(np.uint16)
    ck = oracle.empty_cache(cfg, pairs, 1, w.S)
    cv = oracle.empty_cache(cfg, pairs, 1, w.S)
    t0 = time.perf_counter()
    yk = oracle.quantize_products(cfg, k16, ck, 0, threads)
    yv = oracle.quantize_products(cfg, v16, cv, 0, threads)
    tq = time.perf_counter() - t0
    qsteps = synth.queries(ws, steps=256)
    td, n = 0.0, 0
    while n < 256 and (n == 0 or td < decode_seconds):
        qh = qsteps[n].reshape(-1, G, w.d)[:pairs]          # [pairs, G, d]
        t0 = time.perf_counter()
        kh, _ = oracle.dequantize(cfg, ck, 0, w.S, threads)
        vh, _ = oracle.dequantize(cfg, cv, 0, w.S, threads)
        oracle.attention(np.ascontiguousarray(qh).view(np.uint16).reshape(pairs, G, w.d), kh, vh, None, threads)
        td += time.perf_counter() - t0
        n += 1
    nbytes = (accounting.quantize_bytes(w.d, bits, flags, pairs, 1, w.S)
              + n * accounting.decode_bytes(w.d, bits, flags, pairs, 1, G, w.S))
    return nbytes, tq + td, n, tq, (cfg, ck, cv, yk, yv)


def sampled_parity(w, bits, state, cache, pairs):
    """The GPU cache's prefill blocks of the first `pairs` (batch row, kv
    head) slices against the oracle's: codes bit-exact except at rounding
    half-points (each difference is proven to be one: the oracle's exact
    product lies within 1e-6 of k + 1/2), fp16 side parameters compared in
    ulps."""
    import oracle
    cfg, ck, cv, yk, yv = state
    rb = oracle.row_bytes(w.d, bits)
    res = {"slices": pairs, "tokens_per_slice": w.S, "codes_compared": 0, "code_mismatches": 0,
           "half_point_cases": 0, "non_half_point_mismatches": 0, "max_param_ulp": 0}

    def ulps(a, b):
        key = lambda x: np.where(x.astype(np.int32) & 0x8000, -(x.astype(np.int32) & 0x7FFF), x.astype(np.int32))
        return int(np.max(np.abs(key(a) - key(b)))) if a.size else 0

    for i, (oc, y) in enumerate(((ck, yk), (cv, yv))):
        g = cache.codes[i].reshape(-1, cache.codes[i].shape[2], rb)[:pairs, :w.S].cpu().numpy()
        if i == 1 and w.d == 128:
            g = pairv_rows(g, bits)
        gq, _ = oracle.unpack_rows(g.reshape(-1, rb), w.d, bits)
        oq, _ = oracle.unpack_rows(oc["codes"].reshape(-1, rb), w.d, bits)
        diff = gq.astype(np.int32) - oq.astype(np.int32)
        bad = diff != 0
        hp = oracle.half_point_distance(y.reshape(diff.shape)) <= 1e-6
        res["codes_compared"] += int(diff.size)
        res["code_mismatches"] += int(bad.sum())
        res["half_point_cases"] += int((bad & hp).sum())
        res["non_half_point_mismatches"] += int((bad & ~hp).sum()) + int((np.abs(diff) > 1).sum())
        for name in ("tok", "chan", "off"):
            gt = getattr(cache, name)[i]
            if gt is None or oc[name] is None:
                continue
            n_ = oc[name].shape[2]
            gv = gt.reshape(-1, gt.shape[2], gt.shape[3])[:pairs, :n_].cpu().numpy().view(np.uint16)
            res["max_param_ulp"] = max(res["max_param_ulp"], ulps(gv, oc[name].reshape(gv.shape)))
    return res


def pairv_rows(codes, bits):
    """Pair-interleaved V code rows of head dim 128 (the library's layout,
    include/kvq.h) -> token-major rows, as the oracle stores them."""
    *lead, n, rb = codes.shape
    x = codes.reshape(*lead, n // 2, 2 * rb)
    if bits == 4:
        nch = 2 * rb // 16
        ch = x.reshape(*lead, n // 2, nch, 16)
        k = np.arange(n // 2)[:, None]
        idx = np.arange(nch)[None, :] ^ (2 * (k & 1))
        ch = np.take_along_axis(ch, np.broadcast_to(idx[..., None], ch.shape), axis=-2)
        x = ch.reshape(*lead, n // 2, 2 * rb)
    w4 = x.reshape(*lead, n // 2, rb // 2, 2, 2)
    return np.ascontiguousarray(np.swapaxes(w4, -3, -2)).reshape(*lead, n, rb)


def oracle_sample_text(w, pairs, n, secs):
    return (f"{pairs} (batch row, kv head) slices of the {WORKLOAD} workload ({w.S} prefilled tokens, "
            f"{w.Hq // w.Hkv} query heads each): oracle quantize of the prefill + {n} decode steps "
            f"(dequantize + fp64 attention), {secs:.1f} s")


def rank_workload(rank: int, batch=None, stream=None):
    """The benchmark workload of one rank: every rank runs its own batch of
    the same shape (weak scaling), drawn from a seed of its own."""
    w = synth.WORKLOADS[WORKLOAD].scaled(seed=rank)
    if batch:
        w = w.scaled(B=batch)
    if stream is not None:
        w = w.scaled(stream=stream)
    elif w.stream == 0:
        w = w.scaled(stream=16)  # workloads quoted without streaming: 16 decode steps per step
    return w


def batch_shard(B: int, rank: int, world: int):
    """Batch rows [lo, hi) of rank `rank` when one workload's batch is split
    over `world` ranks: contiguous, sizes differ by at most one row.  Every
    (batch row, kv head) pair is an independent problem, so the shards need
    no collective on the data path."""
    q, r = divmod(B, world)
    lo = rank * q + min(rank, r)
    return lo, lo + q + (1 if rank < r else 0)


def sum_over_ranks(x: float, world: int, device) -> float:
    """The job's total of a per-rank figure (bytes moved by all ranks)."""
    if world == 1:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


def max_over_ranks(ms: float, world: int, device) -> float:
    """The slowest rank's time: the job's step time under weak scaling."""
    if world == 1:
        return ms
    import torch
    t = torch.tensor([ms], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def l2_note(w, bits):
    cache_b = accounting.decode_bytes(w.d, bits, flags_of(MODE), w.B, w.Hkv, w.Hq, w.S)
    prefill_b = 2 * w.B * w.Hkv * w.S * w.d * 2
    if min(cache_b, prefill_b) > 126e6:
        return (f"inputs larger than L2 (packed cache {cache_b / 1e6:.0f} MB, fp16 prefill "
                f"{prefill_b / 2**30:.1f} GiB): no flush needed")
    return (f"packed cache {cache_b / 1e6:.1f} MB, fp16 prefill {prefill_b / 1e6:.1f} MB: what fits in the "
            f"126 MB L2 stays there between calls (no flush)")


def bench_config(w, bits, world, split=False):
    return {"workload": WORKLOAD, "mode": MODE, "bits": bits, "batch": w.B, "q_heads": w.Hq,
            "kv_heads": w.Hkv, "head_dim": w.d, "seq_len": w.S, "streamed": w.stream,
            "l2": l2_note(w, bits),
            "parallelism": (f"batch split over {world} ranks (strong; batch above is per rank, no collective)"
                            if split else f"weak x{world} (independent batches, no collective)")}


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------ reference arm

def run_reference(args, rank: int, world: int):
    if rank != 0:
        return 0
    w = synth.WORKLOADS[WORKLOAD]
    pairs = max(1, min(host_cores(), 32))
    threads = pairs
    for _ in range(args.warmup):
        run_oracle_sample(w, MODE, BITS, pairs, threads, 1.0)
    tot_b, tot_s, tot_n = 0.0, 0.0, 0
    for _ in range(args.steps):
        nb, secs, n, _, _ = run_oracle_sample(w, MODE, BITS, pairs, threads, 4.0)
        tot_b += nb
        tot_s += secs
        tot_n += n
    gbs = tot_b / tot_s / 1e9
    sample = oracle_sample_text(w, pairs, tot_n, tot_s) + f" over {args.steps} steps"
    line = {"impl": "reference", "metric": METRIC, "value": gbs, "unit": "GB/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * tot_s / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": bench_config(w, BITS, world),
            "cpu_baseline": {"value": gbs, "unit": "GB/s", "cores": threads, "kind": "oracle", "sample": sample},
            "e2e": {"value": gbs, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------ our arm

def run_ours(args, rank: int, world: int):
    import torch
    from kv_cache_bit_b200 import kvq

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    split = args.split_batch and world > 1
    # weak scaling: every rank its own draw of the workload; --split-batch:
    # one workload (rank 0's draw) whose batch is split over the ranks
    w = rank_workload(0 if split else rank, args.batch, args.stream)
    BITS = args.bits
    flags = flags_of(MODE)
    G = w.Hq // w.Hkv
    n_stream = w.stream
    cap = ((w.S + n_stream + 127) // 128) * 128

    # inputs, resident before timing
    K, V = synth.kv(w)
    ks, vs = synth.stream_tokens(w)
    qs = synth.queries(w, steps=n_stream)
    if split:
        lo, hi = batch_shard(w.B, rank, world)
        K, V = K[lo:hi], V[lo:hi]
        ks, vs, qs = ks[:, lo:hi], vs[:, lo:hi], qs[:, lo:hi]
        w = w.scaled(B=hi - lo)
    tod = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev)
    Kd, Vd, ksd, vsd, qsd = tod(K), tod(V), tod(ks), tod(vs), tod(qs)
    signs = kvq.kvq_make_signs(synth.SIGN_SEED, w.d) if synth.MODES[MODE][1] else None
    cfg = kvq.Config(w.d, BITS, flags, signs, device=dev)
    cache = kvq.KVCache.allocate(cfg, w.B, w.Hkv, cap, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    ws_bytes = kvq.kvq_decode_workspace_bytes(cfg, cache, w.Hq)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)

    ev = []

    def step(record: bool):
        cache.c.len = 0
        if record:
            e0 = torch.cuda.Event(enable_timing=True); e0.record(stream)
        kvq.kvq_quantize_block(cfg, cache, Kd, Vd, 0, w.S, stream)
        if record:
            e1 = torch.cuda.Event(enable_timing=True); e1.record(stream)
            ev.append(("quantize", e0, e1))
            prev = e1
        for i in range(n_stream):
            kvq.kvq_append_token(cfg, cache, ksd[i], vsd[i], stream)
            if record:
                d0 = torch.cuda.Event(enable_timing=True); d0.record(stream)
                flush = (w.S + i + 1) % 128 == 0
                ev.append(("flush" if flush else "append", prev, d0))
            kvq.kvq_decode_attention(cfg, cache, qsd[i], w.Hq, 0.0, out, ws, ws_bytes, stream)
            if record:
                d1 = torch.cuda.Event(enable_timing=True); d1.record(stream)
                ev.append(("decode", d0, d1))
                prev = d1

    # algorithmic bytes of one step
    step_bytes = accounting.quantize_bytes(w.d, BITS, flags, w.B, w.Hkv, w.S)
    dec_bytes = []
    for i in range(n_stream):
        length = w.S + i + 1  # the decode after append i sees this many tokens
        step_bytes += accounting.append_bytes(w.d, BITS, flags, w.B, w.Hkv, flush=(length % 128 == 0))
        db = accounting.decode_bytes(w.d, BITS, flags, w.B, w.Hkv, w.Hq, length)
        dec_bytes.append(db)
        step_bytes += db
    launches_per_step = 1 + n_stream * (1 + 2)

    for _ in range(args.warmup):
        step(False)
    torch.cuda.synchronize()

    uuid = None
    try:
        uuid = "GPU-" + str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid)
    sampler.start()
    time.sleep(0.5)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    # the timed steps: events only at the two ends (an event between two
    # calls holds back the launch of the second)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for _ in range(args.steps):
        step(False)
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(t_start.elapsed_time(t_end) / args.steps, world, dev)

    # the decode kernels' duration: consecutive calls at the stream's mean
    # cache shape (the last length with 64 residual tokens: 65 blocks + 64
    # tokens for the throughput workload), events around the loop
    final = cache.len
    t_len = next((L for L in range(final, w.S, -1) if L % 128 == 64), final)
    cache.c.len = t_len
    for _ in range(3):
        kvq.kvq_decode_attention(cfg, cache, qsd[n_stream - 1 if n_stream else 0], w.Hq, 0.0, out, ws, ws_bytes,
                                 stream)
    n_dec = 32
    k0 = torch.cuda.Event(enable_timing=True)
    k1 = torch.cuda.Event(enable_timing=True)
    k0.record(stream)
    for _ in range(n_dec):
        kvq.kvq_decode_attention(cfg, cache, qsd[n_stream - 1 if n_stream else 0], w.Hq, 0.0, out, ws, ws_bytes,
                                 stream)
    k1.record(stream)
    torch.cuda.synchronize()
    clocks = sampler.stop()
    k_s = max_over_ranks(k0.elapsed_time(k1) / n_dec, world, dev) / 1e3
    k_bytes = accounting.decode_bytes(w.d, BITS, flags, w.B, w.Hkv, w.Hq, t_len)
    # the quantize kernel's duration: consecutive calls over the prefill
    # (they rewrite the same blocks), events around the loop
    n_q = 3
    q0 = torch.cuda.Event(enable_timing=True)
    q1 = torch.cuda.Event(enable_timing=True)
    cache.c.len = 0
    kvq.kvq_quantize_block(cfg, cache, Kd, Vd, 0, w.S, stream)
    q0.record(stream)
    for _ in range(n_q):
        cache.c.len = 0
        kvq.kvq_quantize_block(cfg, cache, Kd, Vd, 0, w.S, stream)
    q1.record(stream)
    torch.cuda.synchronize()
    qk_s = max_over_ranks(q0.elapsed_time(q1) / n_q, world, dev) / 1e3
    cache.c.len = final

    # one more step with events around every call: where the step's time goes
    # (each event delays the launch behind it, so these spans run long)
    step(True)
    torch.cuda.synchronize()
    q_ms = [a.elapsed_time(b) for k, a, b in ev if k == "quantize"]
    d_ms = [a.elapsed_time(b) for k, a, b in ev if k == "decode"]
    a_ms = [a.elapsed_time(b) for k, a, b in ev if k == "append"]
    f_ms = [a.elapsed_time(b) for k, a, b in ev if k == "flush"]
    dec_avg_bytes = sum(dec_bytes) / len(dec_bytes)
    dec_span_s = (sum(d_ms) / len(d_ms)) / 1e3
    q_avg_s = (sum(q_ms) / len(q_ms)) / 1e3
    q_bytes = accounting.quantize_bytes(w.d, BITS, flags, w.B, w.Hkv, w.S)
    peak, peak_kind = measured_peak_gbs()
    dec_gbs = k_bytes / k_s / 1e9
    q_gbs = q_bytes / qk_s / 1e9
    value = sum_over_ranks(step_bytes, world, dev) / (ms / 1e3) / 1e9

    extra = not (args.no_int2 or world > 1 or BITS != 4 or WORKLOAD != "throughput")
    int2 = run_variant(w, 2, flags, Kd, Vd, ksd, vsd, qsd, stream, peak) if extra else None
    dq = run_variant(w, 4, flags | 16, Kd, Vd, ksd, vsd, qsd, stream, peak) if extra and flags & 4 else None

    # end to end through the public calls, host buffers, copies inside the region
    ref_last = out.clone()  # the last decode output of the device-resident run
    e2e = None if args.no_e2e else run_e2e(args, w, cfg, cache, out, ws, ws_bytes, K, V, ks, vs, qs, stream, dev,
                                           step_bytes, world, ref_last)

    if rank != 0:
        return 0
    line = {
        "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "strong" if split else "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": bench_config(w, BITS, world, split),
        "decode": {"gbs": dec_gbs, "frac_of_hbm": dec_gbs / peak, "us_per_call": k_s * 1e6,
                   "bytes_per_call": k_bytes, "length": t_len,
                   "timing": f"{n_dec} consecutive calls at {t_len} tokens, CUDA events around the loop",
                   "tokens_per_s": world * w.B / k_s,
                   "cache_tokens_per_s": world * w.B * w.Hkv * t_len / k_s,
                   "in_step_us_per_call": dec_span_s * 1e6, "in_step_bytes_per_call": dec_avg_bytes,
                   "in_step_gbs": dec_avg_bytes / dec_span_s / 1e9},
        "append": {"us_per_call": 1e3 * sum(a_ms) / max(1, len(a_ms)),
                   "flush_us_per_call": 1e3 * sum(f_ms) / max(1, len(f_ms)) if f_ms else None,
                   "flushes_per_step": len(f_ms) // max(1, args.steps)},
        "quantize": {"gbs": q_gbs, "frac_of_hbm": q_gbs / peak, "us_per_call": qk_s * 1e6,
                     "bytes_per_call": q_bytes,
                     "timing": f"{n_q} consecutive calls over the prefill, CUDA events around the loop",
                     "in_step_us_per_call": q_avg_s * 1e6},
        "tokens_per_s": world * w.B * n_stream / (ms / 1e3),
        "roofline": {"bound": "hbm", "achieved": dec_gbs, "peak": peak, "unit": "GB/s", "frac": dec_gbs / peak,
                     "traffic": decode_traffic(),
                     "kernel": "kvq_decode_attention (decode + combine launches), per call, consecutive calls",
                     "peak_kind": f"{peak_kind} copy bandwidth (burst)",
                     "traffic_source": "profiles/decode_traffic_throughput.md (ncu dram bytes, one call)"},
        "e2e": e2e,
        "int2": int2,
        "int4_dq": dq,
        "gpu_launches": launches_per_step * args.steps,
        "clocks": clocks,
    }
    if world == 1 and not args.no_cpu_baseline:
        # the oracle on the first slices of this run's own prefill, timed,
        # then (untimed) compared with the GPU cache of the same slices
        pairs = max(1, min(host_cores(), 32))
        data = (K.reshape(-1, 1, w.S, w.d)[:pairs], V.reshape(-1, 1, w.S, w.d)[:pairs])
        nb, secs, n, _, state = run_oracle_sample(w, MODE, BITS, pairs, pairs, 12.0, data)
        line["cpu_baseline"] = {"value": nb / secs / 1e9, "unit": "GB/s", "cores": pairs, "kind": "oracle",
                                "sample": oracle_sample_text(w, pairs, n, secs)}
        line["parity"] = sampled_parity(w, BITS, state, cache, pairs)
    print(json.dumps(line), flush=True)
    return 0


def run_variant(w, bits, flags, Kd, Vd, ksd, vsd, qsd, stream, peak):
    """The same workload with other codes (INT2) or side parameters (DQ):
    quantize of the prefill, the streamed appends, then consecutive decode
    calls at the stream's mean cache shape (the last length with 64 residual
    tokens), CUDA events on the launching stream."""
    import torch
    from kv_cache_bit_b200 import kvq
    dev = Kd.device
    cap = ((w.S + w.stream + 127) // 128) * 128
    cfg = kvq.Config(w.d, bits, flags, None, device=dev)
    cache = kvq.KVCache.allocate(cfg, w.B, w.Hkv, cap, device=dev)
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.float32, device=dev)
    ws_bytes = kvq.kvq_decode_workspace_bytes(cfg, cache, w.Hq)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)
    for _ in range(3):
        cache.c.len = 0
        kvq.kvq_quantize_block(cfg, cache, Kd, Vd, 0, w.S, stream)
    q0, q1 = ev(), ev()
    reps = 3
    q0.record(stream)
    for _ in range(reps):
        cache.c.len = 0
        kvq.kvq_quantize_block(cfg, cache, Kd, Vd, 0, w.S, stream)
    q1.record(stream)
    for i in range(w.stream):
        kvq.kvq_append_token(cfg, cache, ksd[i], vsd[i], stream)
    t_len = next((L for L in range(cache.len, w.S, -1) if L % 128 == 64), cache.len)
    cache.c.len = t_len
    qlast = qsd[w.stream - 1] if w.stream else qsd[0]
    for _ in range(3):
        kvq.kvq_decode_attention(cfg, cache, qlast, w.Hq, 0.0, out, ws, ws_bytes, stream)
    d0, d1 = ev(), ev()
    n = 32
    d0.record(stream)
    for _ in range(n):
        kvq.kvq_decode_attention(cfg, cache, qlast, w.Hq, 0.0, out, ws, ws_bytes, stream)
    d1.record(stream)
    torch.cuda.synchronize()
    q_s = q0.elapsed_time(q1) / reps / 1e3
    d_s = d0.elapsed_time(d1) / n / 1e3
    qb = accounting.quantize_bytes(w.d, bits, flags, w.B, w.Hkv, w.S)
    db = accounting.decode_bytes(w.d, bits, flags, w.B, w.Hkv, w.Hq, t_len)
    return {"quantize": {"gbs": qb / q_s / 1e9, "frac_of_hbm": qb / q_s / 1e9 / peak, "us_per_call": q_s * 1e6,
                         "bytes_per_call": qb},
            "decode": {"gbs": db / d_s / 1e9, "frac_of_hbm": db / d_s / 1e9 / peak, "us_per_call": d_s * 1e6,
                       "bytes_per_call": db, "length": t_len}}


def run_e2e(args, w, cfg, cache, out, ws, ws_bytes, K, V, ks, vs, qs, stream, dev, step_bytes, world, ref_last):
    """Same step through the public calls with pinned HOST inputs: the prefill,
    the streamed tokens and the queries are copied host->device inside the
    timed region, and every decode output is copied back.  The copies run on
    their own streams and overlap the kernels: the prefill moves in batch
    chunks, each quantized as soon as it has landed (kvq_quantize_block on a
    batch-row view of the cache), and the next step's prefill moves while
    this step decodes (its device buffer is free once this step's quantize
    calls have read it); the streamed tokens' inputs of a step move in one
    copy per tensor at its start (double-buffered across steps) and each
    decode output moves back while the next token computes (double buffers,
    ordered by events)."""
    import torch
    from kv_cache_bit_b200 import kvq
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).pin_memory()
    Kh, Vh, ksh, vsh, qsh = pin(K), pin(V), pin(ks), pin(vs), pin(qs)
    Kd = torch.empty_like(Kh, device=dev)
    Vd = torch.empty_like(Vh, device=dev)
    # the streamed tokens' inputs of a whole step, double-buffered across steps
    tokd = [[torch.empty_like(x, device=dev) for x in (ksh, vsh, qsh)] for _ in range(2)]
    outd = [out, torch.empty_like(out)]
    outh = torch.empty((w.stream,) + tuple(out.shape), dtype=torch.float32).pin_memory()
    h2d_s = torch.cuda.Stream(dev)  # streamed-token inputs
    pre_s = torch.cuda.Stream(dev)  # prefill chunks
    d2h_s = torch.cuda.Stream(dev)
    nchunk = 8 if w.B % 8 == 0 else 1
    bc = w.B // nchunk
    views = [cache.rows(c * bc, (c + 1) * bc) for c in range(nchunk)]
    ev = lambda: torch.cuda.Event()
    # events carried across steps: each buffer's last reader or last copy
    tok_free = [None, None]
    out_free = [None, None]
    pre_free = [None]  # the prefill buffer's last reader (the previous step's quantize)
    parity = [0]

    def step():
        tb = parity[0]
        parity[0] ^= 1
        with torch.cuda.stream(h2d_s):
            if tok_free[tb] is not None:
                h2d_s.wait_event(tok_free[tb])
            for dst, src in zip(tokd[tb], (ksh, vsh, qsh)):
                dst.copy_(src, non_blocking=True)
            tok_ready = ev()
            tok_ready.record(h2d_s)
        cache.c.len = 0
        # prefill: chunk c copied on pre_s, quantized on the compute stream
        for c in range(nchunk):
            rows = slice(c * bc, (c + 1) * bc)
            with torch.cuda.stream(pre_s):
                if c == 0 and pre_free[0] is not None:
                    pre_s.wait_event(pre_free[0])
                Kd[rows].copy_(Kh[rows], non_blocking=True)
                Vd[rows].copy_(Vh[rows], non_blocking=True)
                e = ev(); e.record(pre_s)
            stream.wait_event(e)
            views[c].c.len = 0
            kvq.kvq_quantize_block(cfg, views[c], Kd[rows], Vd[rows], 0, w.S, stream)
        pre_free[0] = ev(); pre_free[0].record(stream)
        cache.c.len = w.S

        kd, vd, qd = tokd[tb]
        stream.wait_event(tok_ready)
        for i in range(w.stream):
            j = i % 2
            if out_free[j] is not None:
                stream.wait_event(out_free[j])
            kvq.kvq_append_token(cfg, cache, kd[i], vd[i], stream)
            kvq.kvq_decode_attention(cfg, cache, qd[i], w.Hq, 0.0, outd[j], ws, ws_bytes, stream)
            done = ev(); done.record(stream)
            with torch.cuda.stream(d2h_s):
                d2h_s.wait_event(done)
                outh[i].copy_(outd[j], non_blocking=True)
                out_free[j] = ev(); out_free[j].record(d2h_s)
        tok_free[tb] = ev(); tok_free[tb].record(stream)
        # the step ends when its last output is on the host
        for e in out_free:
            if e is not None:
                stream.wait_event(e)

    step()
    torch.cuda.synchronize()
    steps = max(1, args.steps)
    if world > 1:
        torch.distributed.barrier()
    a = torch.cuda.Event(enable_timing=True)
    b = torch.cuda.Event(enable_timing=True)
    a.record(stream)
    h2d_s.wait_event(a)
    pre_s.wait_event(a)
    d2h_s.wait_event(a)
    for _ in range(steps):
        step()
    b.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(a.elapsed_time(b) / steps, world, dev)
    h2d = (Kh.numel() + Vh.numel()) * 2 + w.stream * (ksh[0].numel() + vsh[0].numel() + qsh[0].numel()) * 2
    d2h = w.stream * out.numel() * 4
    same = bool(torch.equal(outh[w.stream - 1].to(dev), ref_last)) if w.stream else None
    return {"value": world * step_bytes / (ms / 1e3) / 1e9, "unit": "GB/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "overlap": f"copies on three streams; prefill in {nchunk} batch chunks, the next step's prefill "
                       "and streamed-token inputs copied during this step's decode loop",
            "last_output_equals_device_run": same}


def main():
    global WORKLOAD, MODE
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=5)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true", help="skip the end-to-end (host buffers) measurement")
    ap.add_argument("--no-int2", action="store_true", help="skip the INT2 measurement of the same workload")
    ap.add_argument("--split-batch", action="store_true",
                    help="under torchrun: split one workload's batch over the ranks (strong scaling) instead of "
                         "one workload per rank (weak scaling)")
    ap.add_argument("--batch", type=int, default=None, help="override the batch size (smaller profiling cases)")
    ap.add_argument("--stream", type=int, default=None, help="override the number of streamed decode steps")
    ap.add_argument("--bits", type=int, default=BITS, choices=[2, 3, 4])
    ap.add_argument("--workload", default=WORKLOAD, choices=sorted(synth.WORKLOADS),
                    help="another of the five workload configurations (default: the throughput workload)")
    ap.add_argument("--mode", default=None, choices=sorted(synth.MODES), help="quantizer mode (default: the workload's)")
    args = ap.parse_args()
    WORKLOAD = args.workload
    MODE = args.mode or WORKLOAD_MODES[WORKLOAD]

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        return run_ours(args, rank, world)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
