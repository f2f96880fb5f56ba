"""Benchmark of the GEAR KV codec hot path on B200.

One step = one pass over every stage of the path:
  1. encode K and V of a LLaMA-7B-shaped layer (batch 1, 32 heads, 4096
     tokens, d = 128, fp16; 4-bit, group 64, s = 2%, r = 4, T = 3),
  2. one decode-attention step over a compressed cache of batch 16, 32 heads,
     8192 tokens plus the full-precision buffer (fp16, softmax scale 1/sqrt(128)),
  3. appending the new token to that cache (compressing the buffer whenever it
     is full, i.e. every 20th step).
`value` is the encode throughput in GB/s of fp16 KV input; the decode-attention
throughput (tokens/s = sequences per second) is reported beside it. All inputs
are synthetic and seeded (workloads/), resident in HBM before the timed region.
L2 is flushed (a 512 MiB write) before every stage of every timed step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run: every rank runs the same step on
its own data (replicas, no collective on the data path); times are the max
over ranks.
"""
from __future__ import annotations

import argparse
import dataclasses
import json
import math
import os
import statistics
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "KV encode GB/s (fp16 in) + decode-attn tokens/s; % of B200 HBM roofline"
ENC = "llama7b_layer_encode"
DEC = "decode_b16_ctx8192"


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


# DRAM bytes of one decode_warp launch on the decode workload, measured by ncu
# (dram__bytes_read.sum + dram__bytes_write.sum of one launch); set to None
# whenever the kernel changes, until it is captured again.
DECODE_TRAFFIC_BYTES = 830936064 + 7828224


def per_token_bytes(w, meta_f16: bool = False) -> int:
    """Compressed bytes per token of one tensor: codes + (scale, zero) per group
    (binary32 pairs, or binary16 pairs with meta_f16) + outlier index and value + L row."""
    k = math.ceil(w.s * w.d - 1e-9)
    esz = 4 if w.dtype == "f32" else 2
    return (w.d * w.bits // 8 + (w.d // w.group) * (4 if meta_f16 else 8) + k * (1 + esz)
            + w.rank * (4 if w.dtype == "f32" else 2))


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """Polls the GPU's SM clock and clock-event reasons through NVML (read-only
    queries) from a background thread every ~2 ms while the timed region runs."""

    REASONS = {"hw_slowdown": "nvmlClocksEventReasonHwSlowdown",
               "hw_thermal_slowdown": "nvmlClocksEventReasonHwThermalSlowdown",
               "sw_thermal_slowdown": "nvmlClocksEventReasonSwThermalSlowdown",
               "sw_power_cap": "nvmlClocksEventReasonSwPowerCap"}

    def __init__(self, index: int):
        self.index = index
        self.samples = []
        self.reasons = set()
        self.stop_flag = False
        self.thread = None
        self.error = None

    def start(self):
        import threading
        try:
            import pynvml
            pynvml.nvmlInit()
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            idx = int(vis.split(",")[self.index]) if vis else self.index
            self.h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.nv = pynvml
        except Exception as e:  # NVML missing: report it, keep benchmarking
            self.error = str(e)
            return

        def run():
            nv = self.nv
            while not self.stop_flag:
                try:
                    self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                    r = nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
                    for name, attr in self.REASONS.items():
                        if r & getattr(nv, attr):
                            self.reasons.add(name)
                except Exception as e:
                    self.error = str(e)
                    return
                time.sleep(0.002)

        self.thread = threading.Thread(target=run, daemon=True)
        self.thread.start()

    def stop(self) -> dict:
        if self.thread is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
                    "error": self.error or "nvml unavailable"}
        self.stop_flag = True
        self.thread.join()
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ---------------------------------------------------------------- oracle arm
def oracle_encode_gbps(seconds_budget: float = 12.0, units_cap: int = 64):
    """The C oracle encoding units of the LLaMA-7B layer workload on all host
    cores; returns (GB/s of fp16 input, cores, sample description)."""
    import oracle
    import workloads as wl
    from concurrent.futures import ThreadPoolExecutor
    w = wl.WORKLOADS[ENC]
    p = oracle.Params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank, power_iters=w.iters,
                      buffer_len=w.buffer_len, buffer_rank=w.buffer_rank, seed=w.seed)
    cores = os.cpu_count() or 1
    jobs = [(which, h) for h in range(w.H) for which in ("k", "v")][:units_cap]
    inputs = [wl.kv_unit_np(w, which, 0, 0, h) for which, h in jobs]
    t0 = time.perf_counter()
    done = 0
    with ThreadPoolExecutor(max_workers=cores) as ex:
        for i in range(0, len(inputs), cores):
            list(ex.map(lambda x: oracle.encode_unit(x, p), inputs[i:i + cores]))
            done += len(inputs[i:i + cores])
            if time.perf_counter() - t0 > seconds_budget:
                break
    dt = time.perf_counter() - t0
    nbytes = done * w.n * w.d * 2
    return nbytes / dt / 1e9, cores, f"{done} of {2 * w.H} (head, K/V) units of {ENC}, {w.n} tokens each"


def bench_config(world: int) -> dict:
    """The workload both arms report (the reference arm times its encode part)."""
    import workloads as wl
    we, wd = wl.WORKLOADS[ENC], wl.WORKLOADS[DEC]
    return {"workload": f"{ENC} + {DEC}",
            "encode": {"batch": we.B, "heads": we.H, "tokens": we.n, "head_dim": we.d, "bits": we.bits,
                       "group": we.group, "s": we.s, "rank": we.rank, "iters": we.iters},
            "decode": {"batch": wd.B, "heads": wd.H, "context": wd.n, "buffer": wd.buffer_len},
            "l2": "flushed (512 MiB write) before every timed stage", "parallelism": f"replicas x{world}"}


def max_over_ranks(v: float, world: int, device) -> float:
    """The largest of every rank's value (the slowest rank's time). All ranks call
    it in the same order; one all-reduce of a scalar, nothing on the data path."""
    if world == 1:
        return v
    import torch
    t = torch.tensor([v], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    vals = []
    cores, sample = None, None
    for _ in range(args.warmup):
        oracle_encode_gbps(seconds_budget=3.0, units_cap=8)
    step_ms = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        v, cores, sample = oracle_encode_gbps(seconds_budget=6.0, units_cap=16)
        step_ms.append((time.perf_counter() - t0) * 1e3)
        vals.append(v)
    v = statistics.median(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(v, 6), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(statistics.median(step_ms), 3),
            "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32/f64 (oracle)", "data": "synthetic",
            "config": bench_config(world),
            "cpu_baseline": {"value": round(v, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": round(v, 6), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------- GPU arm
def run_gpu(args, rank: int, world: int):
    import torch
    import kv_cache_compression_gear_b200 as gear
    import workloads as wl

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    we, wd = wl.WORKLOADS[ENC], wl.WORKLOADS[DEC]

    def params(w):
        return gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank,
                                power_iters=w.iters, buffer_len=w.buffer_len, buffer_rank=w.buffer_rank,
                                seed=w.seed)

    # ---- encode workload (per-rank layer index so ranks hold different data)
    pe = params(we)
    xk = wl.kv_tensor_torch(we, "k", rank, dev)
    xv = wl.kv_tensor_torch(we, "v", rank, dev)
    enc_k = gear.Cache(pe, we.B, we.H, we.n, 1, torch.float16, dev)
    enc_v = gear.Cache(pe, we.B, we.H, we.n, 1, torch.float16, dev)
    # ---- decode workload: compressed context + full buffer, room for the appends
    pd = params(wd)
    n_steps_total = args.warmup + args.steps + 1
    n_max = wd.n + wd.buffer_len * (2 + n_steps_total // wd.buffer_len)
    nblk = 2 + n_steps_total // wd.buffer_len
    dk = gear.Cache(pd, wd.B, wd.H, n_max, nblk, torch.float16, dev)
    dv = gear.Cache(pd, wd.B, wd.H, n_max, nblk, torch.float16, dev)
    t = wl.kv_tensor_torch(wd, "k", rank, dev)
    dk.encode(t)
    del t
    t = wl.kv_tensor_torch(wd, "v", rank, dev)
    dv.encode(t)
    del t
    for i in range(wd.buffer_fill):
        gear.append_buffer(dk, dv, wl.rows_torch(wd, wl.S_KBUF, rank, i, wd.H, dev),
                           wl.rows_torch(wd, wl.S_VBUF, rank, i, wd.H, dev))
    q = wl.rows_torch(wd, wl.S_Q, rank, 0, wd.Hq, dev)
    new_k = [wl.rows_torch(wd, wl.S_KNEW, rank, i, wd.H, dev) for i in range(n_steps_total)]
    new_v = [wl.rows_torch(wd, wl.S_VNEW, rank, i, wd.H, dev) for i in range(n_steps_total)]
    tau = 1.0 / math.sqrt(128)
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    out = torch.empty((wd.B, wd.Hq, 128), dtype=torch.float16, device=dev)
    torch.cuda.synchronize()

    def reset_encode_caches():
        for c in (enc_k, enc_v):
            c.c.n_comp = c.c.n_buf = c.c.n_blk = c.c.blk0_len = c.c.blk0_rank = 0

    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    step_idx = [0]

    def one_step(record):
        s = step_idx[0]
        step_idx[0] += 1
        reset_encode_caches()
        flush_buf.fill_(s & 0xFF)
        e0, e1 = ev(), ev()
        e0.record()
        gear.encode_batch([enc_k, enc_v], [xk, xv])
        e1.record()
        flush_buf.fill_((s + 1) & 0xFF)
        d0, d1 = ev(), ev()
        d0.record()
        gear.decode_attn(dk, dv, q, tau, out=out)
        d1.record()
        flush_buf.fill_((s + 2) & 0xFF)
        a0, a1 = ev(), ev()
        flushed = dk.n_buf == wd.buffer_len
        a0.record()
        gear.append_buffer(dk, dv, new_k[s], new_v[s])
        a1.record()
        if record is not None:
            record.append((e0, e1, d0, d1, a0, a1, flushed))

    for _ in range(args.warmup):
        one_step(None)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(dev.index)
    clocks.start()
    recs = []
    torch.cuda.synchronize()
    for _ in range(args.steps):
        one_step(recs)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    enc_ms = [r[0].elapsed_time(r[1]) for r in recs]
    dec_ms = [r[2].elapsed_time(r[3]) for r in recs]
    app_ms = [r[4].elapsed_time(r[5]) for r in recs]
    nflush = sum(1 for r in recs if r[6])
    assert gear.device_status() == 0, "device-side error word set"

    # ---- end to end through the public API with host buffers
    hk = xk.cpu().pin_memory()
    hv = xv.cpu().pin_memory()
    hq = q.cpu().pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
    dxk, dxv, dq = torch.empty_like(xk), torch.empty_like(xv), torch.empty_like(q)
    e2e_enc, e2e_dec = [], []
    for _ in range(max(3, args.steps // 2)):
        reset_encode_caches()
        flush_buf.fill_(7)
        a, b, c, d = ev(), ev(), ev(), ev()
        a.record()
        dxk.copy_(hk, non_blocking=True)
        dxv.copy_(hv, non_blocking=True)
        gear.encode_batch([enc_k, enc_v], [dxk, dxv])
        b.record()
        c.record()
        dq.copy_(hq, non_blocking=True)
        gear.decode_attn(dk, dv, dq, tau, out=out)
        hout.copy_(out, non_blocking=True)
        d.record()
        torch.cuda.synchronize()
        e2e_enc.append(a.elapsed_time(b))
        e2e_dec.append(c.elapsed_time(d))

    def maxrank(v):
        return max_over_ranks(v, world, dev)

    enc_t = maxrank(sum(enc_ms) / 1e3)
    dec_t = maxrank(sum(dec_ms) / 1e3)
    app_t = maxrank(sum(app_ms) / 1e3)
    e2e_enc_t = maxrank(statistics.median(e2e_enc) / 1e3)
    e2e_dec_t = maxrank(statistics.median(e2e_dec) / 1e3)
    if rank != 0:
        return

    K = args.steps
    enc_in_bytes = 2 * we.B * we.H * we.n * we.d * 2                  # K and V, fp16
    value = world * K * enc_in_bytes / enc_t / 1e9
    dec_tps = world * K * wd.B / dec_t
    hbm, peak_kind = peaks()
    # algorithmic bytes: encode reads the input once and writes the compressed form once
    enc_alg = 2 * (we.B * we.H * we.n * (we.d * 2 + per_token_bytes(we)) + we.B * we.H * we.d * we.rank * 4)
    n_comp = dk.n_comp
    dec_alg = (2 * wd.B * wd.H * n_comp * per_token_bytes(wd) + 2 * wd.B * wd.H * dk.n_blk * wd.rank * 128 * 4
               + 2 * wd.B * wd.H * wd.buffer_fill * 128 * 2 + 2 * wd.B * wd.Hq * 128 * 2)
    enc_gbs = enc_alg / (enc_t / K) / 1e9
    dec_gbs = dec_alg / (dec_t / K) / 1e9
    dominant = "decode" if dec_t >= enc_t else "encode"
    roof = {"bound": "hbm", "kernel": "gear_decode_attn" if dominant == "decode" else "gear_encode",
            "achieved": round(dec_gbs if dominant == "decode" else enc_gbs, 2), "peak": hbm,
            "unit": "GB/s", "frac": round((dec_gbs if dominant == "decode" else enc_gbs) / hbm, 4),
            "peak_kind": peak_kind,
            "traffic": DECODE_TRAFFIC_BYTES if dominant == "decode" else None}
    other = {"kernel": "gear_encode" if dominant == "decode" else "gear_decode_attn",
             "achieved": round(enc_gbs if dominant == "decode" else dec_gbs, 2),
             "frac": round((enc_gbs if dominant == "decode" else dec_gbs) / hbm, 4)}
    line = {
        "metric": METRIC, "value": round(value, 3), "unit": "GB/s", "n_gpus": world, "steps": K,
        "warmup": args.warmup, "ms_per_step": round((enc_t + dec_t + app_t) / K * 1e3, 4),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f16",
        "data": "synthetic (seeded, workloads/)",
        "config": bench_config(world),
        "decode_tokens_per_s": round(dec_tps, 1),
        "stage_ms": {"encode": round(enc_t / K * 1e3, 4), "decode": round(dec_t / K * 1e3, 4),
                     "append": round(app_t / K * 1e3, 4), "appends_with_flush": nflush},
        "roofline": roof, "roofline_other": other,
        "e2e": {"value": round(world * enc_in_bytes / e2e_enc_t / 1e9, 3), "unit": "GB/s",
                "h2d_bytes_per_step": enc_in_bytes + wd.B * wd.Hq * 128 * 2,
                "d2h_bytes_per_step": wd.B * wd.Hq * 128 * 2,
                "decode_tokens_per_s": round(world * wd.B / e2e_dec_t, 1)},
        "gpu_launches": K * (3 + 2 + 1) + nflush * 3,
        "clocks": clk,
    }
    if world == 1:
        line["gear_l"] = variant_measure(gear, wl, we, wd, dev, max(3, K // 2), hbm, s=0.0)
        line["meta_f16"] = variant_measure(gear, wl, we, wd, dev, max(3, K // 2), hbm, s=we.s, meta_f16=True)
        v, cores, sample = oracle_encode_gbps()
        line["cpu_baseline"] = {"value": round(v, 6), "unit": "GB/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    print(json.dumps(line), flush=True)


def variant_measure(gear, wl, we, wd, dev, reps, hbm, s, meta_f16=False):
    """The same two workloads with another outlier fraction s (s = 0 is the pages'
    GEAR-L: group-wise quantization plus low rank, no outliers) or with binary16
    metadata, timed like the main stages (CUDA events, L2 flushed before each timed
    launch sequence). Reported beside GEAR; not the headline."""
    import torch
    w0e = dataclasses.replace(we, s=s)
    w0d = dataclasses.replace(wd, s=s)

    def params(w):
        return gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank,
                                power_iters=w.iters, buffer_len=w.buffer_len, buffer_rank=w.buffer_rank,
                                seed=w.seed, meta_f16=meta_f16)

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # encode: K and V of the layer in one batched encode
    xs = [wl.kv_tensor_torch(w0e, which, 0, dev) for which in ("k", "v")]
    pe = params(w0e)
    cs = [gear.Cache(pe, w0e.B, w0e.H, w0e.n, 1, torch.float16, dev) for _ in range(2)]
    enc = []
    for it in range(reps + 3):
        for c in cs:
            c.c.n_comp = c.c.n_buf = c.c.n_blk = c.c.blk0_len = c.c.blk0_rank = 0
        flush.fill_(it & 0xFF)
        a, b = ev(), ev()
        a.record()
        gear.encode_batch(cs, xs)
        b.record()
        torch.cuda.synchronize()
        if it >= 3:
            enc.append(a.elapsed_time(b))
    del xs, cs
    # decode: compressed context + full buffer
    pd = params(w0d)
    dk = gear.Cache(pd, w0d.B, w0d.H, w0d.n + w0d.buffer_len, 2, torch.float16, dev)
    dv = gear.Cache(pd, w0d.B, w0d.H, w0d.n + w0d.buffer_len, 2, torch.float16, dev)
    for c, which in ((dk, "k"), (dv, "v")):
        t = wl.kv_tensor_torch(w0d, which, 0, dev)
        c.encode(t)
        del t
    for i in range(w0d.buffer_fill):
        gear.append_buffer(dk, dv, wl.rows_torch(w0d, wl.S_KBUF, 0, i, w0d.H, dev),
                           wl.rows_torch(w0d, wl.S_VBUF, 0, i, w0d.H, dev))
    q = wl.rows_torch(w0d, wl.S_Q, 0, 0, w0d.Hq, dev)
    out = torch.empty((w0d.B, w0d.Hq, 128), dtype=torch.float16, device=dev)
    dec = []
    for it in range(reps + 3):
        flush.fill_(it & 0xFF)
        a, b = ev(), ev()
        a.record()
        gear.decode_attn(dk, dv, q, 1.0 / math.sqrt(128), out=out)
        b.record()
        torch.cuda.synchronize()
        if it >= 3:
            dec.append(a.elapsed_time(b))
    assert gear.device_status() == 0, "device-side error word set"
    enc_ms, dec_ms = statistics.median(enc), statistics.median(dec)
    enc_in = 2 * w0e.B * w0e.H * w0e.n * w0e.d * 2
    ptb = per_token_bytes(w0d, meta_f16)
    dec_alg = (2 * w0d.B * w0d.H * w0d.n * ptb + 2 * w0d.B * w0d.H * w0d.rank * 128 * 4
               + 2 * w0d.B * w0d.H * w0d.buffer_fill * 128 * 2 + 2 * w0d.B * w0d.Hq * 128 * 2)
    return {"s": s, "meta_f16": bool(meta_f16), "encode_ms": round(enc_ms, 4),
            "encode_gbs": round(enc_in / enc_ms / 1e6, 3),
            "decode_ms": round(dec_ms, 4), "decode_tokens_per_s": round(w0d.B / dec_ms * 1e3, 1),
            "decode_hbm_frac": round(dec_alg / dec_ms / 1e6 / hbm, 4),
            "bytes_per_token": ptb}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gear", choices=["gear", "reference"])
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime
        import torch
        torch.cuda.set_device(int(os.environ.get("LOCAL_RANK", 0)))
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_gpu(args, rank, world)
    finally:
        if world > 1:
            import torch
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
