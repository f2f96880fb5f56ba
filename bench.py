"""Benchmark of the GEAR KV codec hot path on B200.

One step = one pass over every stage of the path on one workload:
  1. encode the K and V tensors (outliers, group-wise quantization, power
     iteration of the residual; every layer of the workload, batched),
  2. one decode-attention step over the compressed caches plus their
     full-precision buffers (softmax scale 1/sqrt(128)),
  3. append one new token per layer (compressing a full buffer first).
The headline workload is the 2-bit codec at high batch (batch 64, 32 heads,
8192 tokens, fp16; 2-bit, group 32, s = 5%, r = 8, T = 3), the largest fp16
configuration: `value` is its encode throughput in GB/s of fp16 KV input, and
its decode-attention throughput (tokens/s = sequences per second) is reported
beside it. The same fields follow under "configs" for the Llama-3-8B-shaped GQA
cache (32 layers, bf16, 32768 tokens, 20-token buffer) and for the Llama-7B
layer encode with the batch-16, 8192-token decode. All inputs are synthetic
and seeded (workloads/), resident in HBM before the timed region. L2 is flushed
(a 512 MiB write) before every stage of every timed step.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run: every rank runs the same step on
its own data (replicas, no collective on the data path); times are the max
over ranks. --batch-override B runs only the headline workload at batch B, the
small case that counter captures use (its line is not a benchmark value).
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


NOMINAL_HBM_GBS = 8000.0   # the B200's nominal HBM3e bandwidth, beside the measured copy bandwidth


def peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


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


# ---------------------------------------------------------------- scenarios
@dataclasses.dataclass(frozen=True)
class Scenario:
    """One benchmark line: the encode workload, the decode workload (the same one
    when the step decodes the cache it has just encoded) and its name."""
    name: str
    enc: str
    dec: str

    @property
    def same(self) -> bool:
        return self.enc == self.dec


HEADLINE = Scenario("twobit_b64_ctx8192", "twobit_b64_ctx8192", "twobit_b64_ctx8192")
BESIDE = [Scenario("llama3_8b_gqa", "llama3_8b_gqa", "llama3_8b_gqa"),
          Scenario(f"{ENC} + {DEC}", ENC, DEC)]


def scenario_config(sc: Scenario, world: int, batch_override: int | None = None) -> dict:
    import workloads as wl
    we, wd = wl.WORKLOADS[sc.enc], wl.WORKLOADS[sc.dec]

    def desc(w, enc):
        d = {"layers": w.layers, "batch": batch_override or w.B, "kv_heads": w.H, "q_heads": w.Hq,
             "tokens" if enc else "context": w.n, "head_dim": w.d, "dtype": w.dtype, "bits": w.bits,
             "group": w.group, "s": w.s, "rank": w.rank, "iters": w.iters}
        if not enc:
            d["buffer"] = w.buffer_fill
        return d

    cfg = {"workload": sc.name, "encode": desc(we, True), "decode": desc(wd, False),
           "l2": "flushed (512 MiB write) before every timed stage; inputs of the two large configs exceed L2",
           "parallelism": f"replicas x{world}"}
    if batch_override:
        cfg["batch_override"] = batch_override
    return cfg


def bench_config(world: int) -> dict:
    """The headline workload both arms report."""
    return scenario_config(HEADLINE, world)


# ---------------------------------------------------------------- oracle arm
def _oparams(w):
    import oracle
    return oracle.Params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank, power_iters=w.iters,
                         buffer_len=w.buffer_len, buffer_rank=w.buffer_rank, seed=w.seed)


def _sample_units(w, count):
    """(which, layer, b, h) of `count` units spread over the workload, K and V alternating."""
    total = w.layers * w.B * w.H
    out = []
    for i in range(count):
        u = (i * 7919) % total
        layer, rem = divmod(u, w.B * w.H)
        out.append(("k" if i % 2 == 0 else "v", layer, rem // w.H, rem % w.H))
    return out


def oracle_encode_gbps(wname: str, seconds_budget: float = 8.0, units_cap: int = 32, threads: int | None = None):
    """The C oracle encoding a bounded sample of units of a workload on `threads`
    host threads (all cores by default); returns (GB/s of KV input, threads, sample
    description). The sample's throughput stands for the whole workload's (all units
    cost the same)."""
    import oracle
    import workloads as wl
    from concurrent.futures import ThreadPoolExecutor
    w = wl.WORKLOADS[wname]
    p = _oparams(w)
    cores = threads or os.cpu_count() or 1
    jobs = _sample_units(w, units_cap)
    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        inputs = list(ex.map(lambda j: wl.kv_unit_np(w, *j), jobs))
    esz = 4 if w.dtype == "f32" else 2
    t0 = time.perf_counter()
    done = 0
    with ThreadPoolExecutor(max_workers=cores) as ex:
        for i in range(0, len(inputs), cores):
            list(ex.map(lambda x: oracle.encode_unit(x, p), inputs[i:i + cores]))
            done += len(inputs[i:i + cores])
            if time.perf_counter() - t0 > seconds_budget:
                break
    dt = time.perf_counter() - t0
    nbytes = done * w.n * w.d * esz
    return nbytes / dt / 1e9, cores, f"{done} units of {wname} ({w.n} tokens each), extrapolated"


def oracle_decode_tps(wname: str, seconds_budget: float = 4.0, units_cap: int = 16, threads: int | None = None):
    """The C oracle's decode attention (reconstruct K and V of a unit from its
    encoding, then softmax attention for every query head of the unit) on a bounded
    sample of units, scaled to a whole decode step of the workload (all layers,
    batches and kv heads); returns (tokens/s = sequences per second, threads, sample)."""
    import numpy as np
    import oracle
    import workloads as wl
    from concurrent.futures import ThreadPoolExecutor
    w = wl.WORKLOADS[wname]
    p = _oparams(w)
    cores = threads or os.cpu_count() or 1
    hq = w.Hq // w.H
    jobs = [(layer, b, h) for (_, layer, b, h) in _sample_units(w, units_cap)]

    def prep(j):
        layer, b, h = j
        return (oracle.encode_unit(wl.kv_unit_np(w, "k", layer, b, h), p),
                oracle.encode_unit(wl.kv_unit_np(w, "v", layer, b, h), p),
                wl.rows_np(w, wl.S_Q, layer, 0, w.Hq)[b, h * hq:(h + 1) * hq])

    with ThreadPoolExecutor(max_workers=os.cpu_count() or 1) as ex:
        enc = list(ex.map(prep, jobs))
    tau = 1.0 / math.sqrt(w.d)

    def dec(e):
        ku, vu, q = e
        K = oracle.reconstruct_unit(ku, p)
        V = oracle.reconstruct_unit(vu, p)
        return [oracle.attention(q[j], K, V, tau) for j in range(q.shape[0])]

    t0 = time.perf_counter()
    done = 0
    with ThreadPoolExecutor(max_workers=cores) as ex:
        for i in range(0, len(enc), cores):
            list(ex.map(dec, enc[i:i + cores]))
            done += len(enc[i:i + cores])
            if time.perf_counter() - t0 > seconds_budget:
                break
    dt = time.perf_counter() - t0
    units_per_step = w.layers * w.B * w.H
    step_s = dt / done * units_per_step
    np.asarray(0)
    return w.B / step_s, cores, f"{done} units of {wname} (K and V reconstructed, {hq} query heads each), scaled to {units_per_step} units per step"


def cpu_baseline(sc: Scenario) -> dict:
    enc_all, cores, enc_sample = oracle_encode_gbps(sc.enc)
    enc_one, _, enc_sample1 = oracle_encode_gbps(sc.enc, seconds_budget=2.0, units_cap=2, threads=1)
    dec_all, _, dec_sample = oracle_decode_tps(sc.dec)
    dec_one, _, _ = oracle_decode_tps(sc.dec, seconds_budget=1.0, units_cap=2, threads=1)
    return {"value": round(enc_all, 6), "unit": "GB/s", "cores": cores, "kind": "oracle", "sample": enc_sample,
            "single_thread": {"value": round(enc_one, 6), "unit": "GB/s", "cores": 1, "sample": enc_sample1},
            "decode": {"value": round(dec_all, 3), "unit": "tokens/s", "cores": cores, "sample": dec_sample,
                       "single_thread": round(dec_one, 3)}}


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
        oracle_encode_gbps(HEADLINE.enc, seconds_budget=2.0, units_cap=4)
    step_ms = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        v, cores, sample = oracle_encode_gbps(HEADLINE.enc, seconds_budget=4.0, units_cap=16)
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
def _gparams(gear, w, meta_f16=False):
    return gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank, power_iters=w.iters,
                            buffer_len=w.buffer_len, buffer_rank=w.buffer_rank, seed=w.seed, meta_f16=meta_f16)


def enc_alg_bytes(w, n_tensors: int) -> int:
    """Algorithmic bytes of encoding n_tensors tensors shaped like w: the input
    read once, the compressed tokens and the Rf rows written once."""
    esz = 4 if w.dtype == "f32" else 2
    units = w.B * w.H
    return n_tensors * units * (w.n * (w.d * esz + per_token_bytes(w)) + w.d * ((w.rank + 3) // 4 * 4) * 4)


def dec_alg_bytes(w, n_comp: int, n_blk: int, n_buf: int, layers: int) -> int:
    """Algorithmic bytes of one decode step: K and V compressed tokens, their Rf
    rows and buffers read once, q read and the output written once."""
    esz = 4 if w.dtype == "f32" else 2
    units = w.B * w.H
    rp = (max(w.rank, w.buffer_rank) + 3) // 4 * 4
    per_layer = (2 * units * n_comp * per_token_bytes(w) + 2 * units * n_blk * rp * 128 * 4
                 + 2 * units * n_buf * 128 * esz + 2 * w.B * w.Hq * 128 * esz)
    return layers * per_layer


class Runner:
    """Holds the device state of one scenario and runs its steps."""

    def __init__(self, gear, wl, sc: Scenario, dev, rank: int, n_steps_total: int, batch_override=None,
                 layers_override=None):
        import torch
        self.gear, self.wl, self.sc, self.dev = gear, wl, sc, dev
        we, wd = wl.WORKLOADS[sc.enc], wl.WORKLOADS[sc.dec]
        if batch_override:
            we = dataclasses.replace(we, B=batch_override)
            wd = dataclasses.replace(wd, B=batch_override) if not sc.same else we
        if layers_override:
            we = dataclasses.replace(we, layers=layers_override)
            wd = dataclasses.replace(wd, layers=layers_override) if not sc.same else we
        self.we, self.wd = we, wd
        dt = wl.torch_dtype(we.dtype)
        # ---- encode inputs and caches (per layer: K and V); rank r selects the data
        pe = _gparams(gear, we)
        L = we.layers
        if sc.same:
            n_max, nblk = we.n + 2 * we.buffer_len, 2
        else:
            n_max, nblk = we.n, 1
        self.x, self.enc = [], []
        for layer in range(L):
            for which in ("k", "v"):
                self.x.append(wl.kv_tensor_torch(we, which, rank * L + layer, dev))
                self.enc.append(gear.Cache(pe, we.B, we.H, n_max, nblk, dt, dev))
        if sc.same:
            self.dk, self.dv = self.enc[0::2], self.enc[1::2]
        else:
            # persistent decode caches: compressed context + full buffer, room for the appends
            pd = _gparams(gear, wd)
            n_max = wd.n + wd.buffer_len * (2 + n_steps_total // wd.buffer_len)
            nblk = 2 + n_steps_total // wd.buffer_len
            self.dk, self.dv = [], []
            for layer in range(wd.layers):
                kc = gear.Cache(pd, wd.B, wd.H, n_max, nblk, dt, dev)
                vc = gear.Cache(pd, wd.B, wd.H, n_max, nblk, dt, dev)
                for c, which in ((kc, "k"), (vc, "v")):
                    t = wl.kv_tensor_torch(wd, which, rank * wd.layers + layer, dev)
                    c.encode(t)
                    del t
                self.dk.append(kc)
                self.dv.append(vc)
                self.fill_buffer(layer, rank)
        self.q = [wl.rows_torch(wd, wl.S_Q, rank * wd.layers + layer, 0, wd.Hq, dev) for layer in range(wd.layers)]
        self.new_k = [[wl.rows_torch(wd, wl.S_KNEW, rank * wd.layers + layer, i, wd.H, dev)
                       for i in range(n_steps_total)] for layer in range(wd.layers)]
        self.new_v = [[wl.rows_torch(wd, wl.S_VNEW, rank * wd.layers + layer, i, wd.H, dev)
                       for i in range(n_steps_total)] for layer in range(wd.layers)]
        self.out = [torch.empty((wd.B, wd.Hq, 128), dtype=dt, device=dev) for _ in range(wd.layers)]
        self.flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
        self.tau = 1.0 / math.sqrt(128)
        self.rank = rank
        self.step_idx = 0
        torch.cuda.synchronize()

    def fill_buffer(self, layer, rank):
        wl, wd = self.wl, self.wd
        for i in range(wd.buffer_fill):
            self.gear.append_buffer(self.dk[layer], self.dv[layer],
                                    wl.rows_torch(wd, wl.S_KBUF, rank * wd.layers + layer, i, wd.H, self.dev),
                                    wl.rows_torch(wd, wl.S_VBUF, rank * wd.layers + layer, i, wd.H, self.dev))

    def encode(self, xs=None):
        for c in self.enc:
            c.reset()
        self.gear.encode_batch(self.enc, xs or self.x)

    def decode(self, qs=None):
        for layer in range(self.wd.layers):
            self.gear.decode_attn(self.dk[layer], self.dv[layer], (qs or self.q)[layer], self.tau,
                                  out=self.out[layer])

    def step(self, record):
        """encode, (buffer fill, untimed), decode, append; CUDA events around each stage."""
        import torch
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        s = self.step_idx
        self.step_idx += 1
        self.flush.fill_(s & 0xFF)
        e0, e1 = ev(), ev()
        e0.record()
        self.encode()
        e1.record()
        if self.sc.same:
            for layer in range(self.wd.layers):
                self.fill_buffer(layer, self.rank)
        self.flush.fill_((s + 1) & 0xFF)
        d0, d1 = ev(), ev()
        d0.record()
        self.decode()
        d1.record()
        self.flush.fill_((s + 2) & 0xFF)
        flushed = self.dk[0].n_buf == self.wd.buffer_len
        a0, a1 = ev(), ev()
        a0.record()
        for layer in range(self.wd.layers):
            self.gear.append_buffer(self.dk[layer], self.dv[layer], self.new_k[layer][s], self.new_v[layer][s])
        a1.record()
        if record is not None:
            record.append((e0, e1, d0, d1, a0, a1, flushed))

    def launches_per_step(self, flushed: bool) -> int:
        n_enc = len(self.enc)
        enc = 3 * ((n_enc + 15) // 16)
        dec = 2 * self.wd.layers
        app = self.wd.layers * (1 + (3 if flushed else 0))
        return enc + dec + app

    def e2e(self, reps: int):
        """Encode and decode through the public API with the inputs in pinned host
        memory: host-to-device copies inside the timed region, the attention output
        read back to the host. Returns (encode s, decode s, h2d bytes, d2h bytes) or
        None when the host cannot hold a pinned copy of the inputs."""
        import torch
        in_bytes = sum(x.numel() * x.element_size() for x in self.x)
        try:
            import psutil
            avail = psutil.virtual_memory().available
        except Exception:
            avail = 0
        if avail < 2 * in_bytes + (16 << 30):
            return None
        hx = [torch.empty(x.shape, dtype=x.dtype, pin_memory=True) for x in self.x]
        for h, x in zip(hx, self.x):
            h.copy_(x)
        hq = [torch.empty(q.shape, dtype=q.dtype, pin_memory=True) for q in self.q]
        for h, q in zip(hq, self.q):
            h.copy_(q)
        hout = [torch.empty(o.shape, dtype=o.dtype, pin_memory=True) for o in self.out]
        dx = [torch.empty_like(x) for x in self.x]
        dq = [torch.empty_like(q) for q in self.q]
        ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
        te, td = [], []
        for it in range(reps + 1):
            self.flush.fill_(7)
            a, b, c, d = ev(), ev(), ev(), ev()
            a.record()
            for h, x in zip(hx, dx):
                x.copy_(h, non_blocking=True)
            self.encode(dx)
            b.record()
            if self.sc.same:
                for layer in range(self.wd.layers):
                    self.fill_buffer(layer, self.rank)
            c.record()
            for h, q in zip(hq, dq):
                q.copy_(h, non_blocking=True)
            self.decode(dq)
            for h, o in zip(hout, self.out):
                h.copy_(o, non_blocking=True)
            d.record()
            torch.cuda.synchronize()
            if it > 0:
                te.append(a.elapsed_time(b) / 1e3)
                td.append(c.elapsed_time(d) / 1e3)
        del dx, hx
        h2d = in_bytes + sum(q.numel() * q.element_size() for q in self.q)
        d2h = sum(o.numel() * o.element_size() for o in self.out)
        return statistics.median(te), statistics.median(td), h2d, d2h


# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of a
# stage's dominant kernel, from one ncu capture each (profiles/), keyed by
# (scenario, stage); an entry is removed whenever its kernel changes, until it is
# captured again.
# The 2-bit batch-64 workload's traffic comes from a capture of the same step at
# batch 4 (1/16 of the units), scaled by 16: every kernel's traffic is per unit.
TRAFFIC_BYTES = {
    # encode stage: E1 539130624 + 175976960, E2 26284032, E3 723844864 + 30014208 bytes at batch 4
    ("twobit_b64_ctx8192", "encode"): 16 * (539130624 + 175976960 + 26284032 + 723844864 + 30014208),
    # decode_warp 213763840 + 762624 bytes at batch 4
    ("twobit_b64_ctx8192", "decode"): 16 * (213763840 + 762624),
}


def measure(gear, wl, sc: Scenario, dev, rank, world, steps, warmup, hbm, peak_kind, batch_override=None,
            with_e2e=True, layers_override=None):
    import torch
    runner = Runner(gear, wl, sc, dev, rank, warmup + steps + 1, batch_override, layers_override)
    we, wd = runner.we, runner.wd
    for _ in range(warmup):
        runner.step(None)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clocks = ClockSampler(dev.index)
    clocks.start()
    recs = []
    torch.cuda.synchronize()
    for _ in range(steps):
        runner.step(recs)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    assert gear.device_status() == 0, "device-side error word set"
    enc_t = max_over_ranks(sum(r[0].elapsed_time(r[1]) for r in recs) / 1e3, world, dev)
    dec_t = max_over_ranks(sum(r[2].elapsed_time(r[3]) for r in recs) / 1e3, world, dev)
    app_t = max_over_ranks(sum(r[4].elapsed_time(r[5]) for r in recs) / 1e3, world, dev)
    nflush = sum(1 for r in recs if r[6])
    launches = sum(runner.launches_per_step(r[6]) for r in recs)
    n_comp, n_blk, n_buf = runner.dk[0].n_comp, runner.dk[0].n_blk, runner.dk[0].n_buf
    ee = runner.e2e(max(3, steps // 4)) if with_e2e else "not measured for this case"
    if isinstance(ee, tuple):
        ee = tuple(max_over_ranks(v, world, dev) for v in ee[:2]) + ee[2:]
    del runner
    torch.cuda.empty_cache()

    K = steps
    esz = 4 if we.dtype == "f32" else 2
    n_enc_tensors = 2 * we.layers
    enc_in = n_enc_tensors * we.B * we.H * we.n * we.d * esz
    # algorithmic bytes as the decode stage saw them: before the step's append
    # (the step's own append always follows its decode)
    if sc.same:
        dec_alg = dec_alg_bytes(wd, wd.n, 1, wd.buffer_fill, wd.layers)
    else:
        dec_alg = dec_alg_bytes(wd, n_comp, n_blk, n_buf, wd.layers)
    enc_alg = enc_alg_bytes(we, n_enc_tensors)
    enc_gbs = enc_alg / (enc_t / K) / 1e9
    dec_gbs = dec_alg / (dec_t / K) / 1e9
    stages = {"encode": (enc_t, enc_gbs, "gear_encode"), "decode": (dec_t, dec_gbs, "gear_decode_attn")}
    dom = "decode" if dec_t >= enc_t else "encode"
    oth = "encode" if dom == "decode" else "decode"
    roof = {"bound": "hbm", "kernel": stages[dom][2], "achieved": round(stages[dom][1], 2), "peak": hbm,
            "unit": "GB/s", "frac": round(stages[dom][1] / hbm, 4), "peak_kind": peak_kind,
            "frac_nominal": round(stages[dom][1] / NOMINAL_HBM_GBS, 4),
            "traffic": TRAFFIC_BYTES.get((sc.name, dom)),
            "algorithmic_bytes": enc_alg if dom == "encode" else dec_alg}
    other = {"kernel": stages[oth][2], "achieved": round(stages[oth][1], 2), "frac": round(stages[oth][1] / hbm, 4),
             "frac_nominal": round(stages[oth][1] / NOMINAL_HBM_GBS, 4),
             "traffic": TRAFFIC_BYTES.get((sc.name, oth)),
             "algorithmic_bytes": enc_alg if oth == "encode" else dec_alg}
    res = {
        "value": round(world * K * enc_in / enc_t / 1e9, 3), "unit": "GB/s",
        "ms_per_step": round((enc_t + dec_t + app_t) / K * 1e3, 4),
        "decode_tokens_per_s": round(world * K * wd.B / dec_t, 1),
        "stage_ms": {"encode": round(enc_t / K * 1e3, 4), "decode": round(dec_t / K * 1e3, 4),
                     "append": round(app_t / K * 1e3, 4), "appends_with_flush": nflush},
        "roofline": roof, "roofline_other": other,
        "gpu_launches": launches, "clocks": clk,
    }
    if isinstance(ee, tuple):
        te, td, h2d, d2h = ee
        res["e2e"] = {"value": round(world * enc_in / te / 1e9, 3), "unit": "GB/s", "h2d_bytes_per_step": h2d,
                      "d2h_bytes_per_step": d2h, "decode_tokens_per_s": round(world * wd.B / td, 1)}
    else:
        res["e2e"] = {"value": None, "unit": "GB/s",
                      "skipped": ee or "host memory cannot hold a pinned copy of the inputs"}
    return res


def run_gpu(args, rank: int, world: int):
    import torch
    import kv_cache_compression_gear_b200 as gear
    import workloads as wl

    dev = torch.device("cuda", int(os.environ.get("LOCAL_RANK", 0)))
    torch.cuda.set_device(dev)
    hbm, peak_kind = peaks()
    if args.profile_case:
        sc = [b for b in BESIDE if b.enc == args.profile_case][0]
        res = measure(gear, wl, sc, dev, rank, world, args.steps, args.warmup, hbm, peak_kind,
                      layers_override=2 if sc.enc == "llama3_8b_gqa" else None, with_e2e=False)
        if rank == 0:
            print(json.dumps({"profile_case": scenario_config(sc, world), **res}), flush=True)
        return
    if args.batch_override:
        # a smaller batch of the headline workload, for counter captures only (not a bench value)
        res = measure(gear, wl, HEADLINE, dev, rank, world, args.steps, args.warmup, hbm, peak_kind,
                      batch_override=args.batch_override, with_e2e=False)
        if rank == 0:
            print(json.dumps({"profile_case": scenario_config(HEADLINE, world, args.batch_override), **res}),
                  flush=True)
        return
    head = measure(gear, wl, HEADLINE, dev, rank, world, args.steps, args.warmup, hbm, peak_kind)
    beside = {}
    for sc in BESIDE:
        beside[sc.name] = measure(gear, wl, sc, dev, rank, world, max(3, args.steps // 2), 3, hbm, peak_kind)
        beside[sc.name]["config"] = scenario_config(sc, world)
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f16", "data": "synthetic (seeded, workloads/)",
        "config": bench_config(world),
        **{k: v for k, v in head.items() if k not in ("value", "unit", "ms_per_step")},
        "configs": beside,
    }
    if world == 1:
        we, wd = wl.WORKLOADS[ENC], wl.WORKLOADS[DEC]
        line["gear_l"] = variant_measure(gear, wl, we, wd, dev, max(3, args.steps // 2), hbm, s=0.0)
        line["meta_f16"] = variant_measure(gear, wl, we, wd, dev, max(3, args.steps // 2), hbm, s=we.s,
                                           meta_f16=True)
        line["kivi_keys"] = variant_measure(gear, wl, we, wd, dev, max(3, args.steps // 2), hbm, s=we.s,
                                            kivi=True)
        line["paged"] = paged_measure(gear, wl, wl.WORKLOADS[DEC], dev, max(3, args.steps // 2), hbm)
        line["cpu_baseline"] = cpu_baseline(HEADLINE)
        for sc in BESIDE:
            line["configs"][sc.name]["cpu_baseline"] = cpu_baseline(sc)
    print(json.dumps(line), flush=True)


def variant_measure(gear, wl, we, wd, dev, reps, hbm, s, meta_f16=False, kivi=False):
    """The same two workloads with another outlier fraction s (s = 0 is the pages'
    GEAR-L: group-wise quantization plus low rank, no outliers), with binary16
    metadata, or (kivi) with the KIVI-combined keys (per-channel groups of g tokens;
    values per token; a buffer of whole groups), timed like the main stages (CUDA
    events, L2 flushed before each timed launch sequence). Reported beside GEAR;
    not the headline."""
    import torch
    w0e = dataclasses.replace(we, s=s)
    w0d = dataclasses.replace(wd, s=s)
    if kivi:   # the buffer holds whole key groups
        w0e = dataclasses.replace(w0e, buffer_len=we.group)
        w0d = dataclasses.replace(w0d, buffer_len=wd.group)

    def params(w, which="v"):
        return gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank,
                                power_iters=w.iters, buffer_len=w.buffer_len, buffer_rank=w.buffer_rank,
                                seed=w.seed, meta_f16=meta_f16, channel_groups=kivi and which == "k")

    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    # encode: K and V of the layer in one batched encode (two encodes when the
    # keys take per-channel groups: the batch wants one parameter set)
    xs = [wl.kv_tensor_torch(w0e, which, 0, dev) for which in ("k", "v")]
    cs = [gear.Cache(params(w0e, which), w0e.B, w0e.H, w0e.n, 1, torch.float16, dev) for which in ("k", "v")]
    enc = []
    for it in range(reps + 3):
        for c in cs:
            c.reset()
        flush.fill_(it & 0xFF)
        a, b = ev(), ev()
        a.record()
        if kivi:
            for c, x in zip(cs, xs):
                c.encode(x)
        else:
            gear.encode_batch(cs, xs)
        b.record()
        torch.cuda.synchronize()
        if it >= 3:
            enc.append(a.elapsed_time(b))
    del xs, cs
    # decode: compressed context + full buffer
    dk = gear.Cache(params(w0d, "k"), w0d.B, w0d.H, w0d.n + w0d.buffer_len, 2, torch.float16, dev)
    dv = gear.Cache(params(w0d, "v"), w0d.B, w0d.H, w0d.n + w0d.buffer_len, 2, torch.float16, dev)
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
    if kivi:   # keys: per-channel (scale, zero) of a token group instead of per-token groups
        ptb_k = ptb - (w0d.d // w0d.group) * 8 + (w0d.d * 8) // w0d.group
        dec_alg = (w0d.B * w0d.H * w0d.n * (ptb + ptb_k) + 2 * w0d.B * w0d.H * w0d.rank * 128 * 4
                   + 2 * w0d.B * w0d.H * w0d.buffer_fill * 128 * 2 + 2 * w0d.B * w0d.Hq * 128 * 2)
    return {"s": s, "meta_f16": bool(meta_f16), "kivi_keys": bool(kivi), "encode_ms": round(enc_ms, 4),
            "encode_gbs": round(enc_in / enc_ms / 1e6, 3),
            "decode_ms": round(dec_ms, 4), "decode_tokens_per_s": round(w0d.B / dec_ms * 1e3, 1),
            "decode_hbm_frac": round(dec_alg / dec_ms / 1e6 / hbm, 4),
            "bytes_per_token": ptb}


def paged_measure(gear, wl, wd, dev, reps, hbm, page_tokens=256):
    """The decode workload in the paged layout (gear_encode_rows, gear_append_rows,
    decode through the block table): first with every row at the full context, the
    case the contiguous decode stage times, then with the rows' prompts spread evenly
    over [n/2, n] (each row encoded at its own length). Timed like the main stages
    (CUDA events, L2 flushed before each timed launch sequence). The decode split
    runs over the tokens the rows hold, so both fractions count the tokens read."""
    import torch
    dt = wl.torch_dtype(wd.dtype)
    p = _gparams(gear, wd)
    P = page_tokens
    ppr = -(-(wd.n + 2 * wd.buffer_len) // P)
    nblk = 4
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    ev = lambda: torch.cuda.Event(enable_timing=True)  # noqa: E731
    esz = 4 if wd.dtype == "f32" else 2
    rows = list(range(wd.B))
    xs = {which: wl.kv_tensor_torch(wd, which, 0, dev) for which in ("k", "v")}
    q = wl.rows_torch(wd, wl.S_Q, 0, 0, wd.Hq, dev)
    out = torch.empty((wd.B, wd.Hq, 128), dtype=dt, device=dev)
    tau = 1.0 / math.sqrt(128)
    kc = gear.PagedCache(p, wd.B, wd.H, P, wd.B * ppr, ppr, nblk, dt, dev)
    vc = gear.PagedCache(p, wd.B, wd.H, P, wd.B * ppr, ppr, nblk, dt, dev)

    def fill(lengths):
        for c in (kc, vc):
            c.release_rows(rows)
        by_len = {}
        for b, n in enumerate(lengths):
            by_len.setdefault(n, []).append(b)
        for n, rs in by_len.items():
            for c, which in ((kc, "k"), (vc, "v")):
                c.encode_rows(rs, xs[which][rs][:, :, :n].contiguous())
        for i in range(wd.buffer_fill):
            gear.append_rows(kc, vc, rows, wl.rows_torch(wd, wl.S_KBUF, 0, i, wd.H, dev),
                             wl.rows_torch(wd, wl.S_VBUF, 0, i, wd.H, dev))

    def time_decode():
        ts = []
        for it in range(reps + 3):
            flush.fill_(it & 0xFF)
            a, b = ev(), ev()
            a.record()
            gear.decode_attn(kc, vc, q, tau, out=out)
            b.record()
            torch.cuda.synchronize()
            if it >= 3:
                ts.append(a.elapsed_time(b))
        return statistics.median(ts)

    def alg_bytes(lengths):
        rp = (max(wd.rank, wd.buffer_rank) + 3) // 4 * 4
        return sum(2 * wd.H * (n * per_token_bytes(wd) + rp * 128 * 4 + wd.buffer_fill * 128 * esz)
                   for n in lengths) + 2 * wd.B * wd.Hq * 128 * esz

    # encode_rows of the whole batch (K and V): the codec on a staging copy, then the scatter into pages
    enc = []
    for it in range(reps + 3):
        for c in (kc, vc):
            c.release_rows(rows)
        flush.fill_(it & 0xFF)
        a, b = ev(), ev()
        a.record()
        kc.encode_rows(rows, xs["k"])
        vc.encode_rows(rows, xs["v"])
        b.record()
        torch.cuda.synchronize()
        if it >= 3:
            enc.append(a.elapsed_time(b))
    full = [wd.n] * wd.B
    fill(full)
    dec_full = time_decode()
    ragged = [wd.n // 2 + (wd.n // 2) * b // max(1, wd.B - 1) // 32 * 32 for b in range(wd.B)]
    fill(ragged)
    dec_rag = time_decode()
    assert gear.device_status() == 0, "device-side error word set"
    enc_ms = statistics.median(enc)
    enc_in = 2 * wd.B * wd.H * wd.n * wd.d * esz
    af, ar = alg_bytes(full), alg_bytes(ragged)
    return {"page_tokens": P, "pages_per_row": ppr, "encode_rows_ms": round(enc_ms, 4),
            "encode_rows_gbs": round(enc_in / enc_ms / 1e6, 3),
            "decode_ms": round(dec_full, 4), "decode_tokens_per_s": round(wd.B / dec_full * 1e3, 1),
            "decode_hbm_frac": round(af / dec_full / 1e6 / hbm, 4),
            "ragged": {"prefill_lengths": [min(ragged), max(ragged)], "decode_ms": round(dec_rag, 4),
                       "decode_hbm_frac": round(ar / dec_rag / 1e6 / hbm, 4)}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="gear", choices=["gear", "reference"])
    ap.add_argument("--batch-override", type=int, default=None,
                    help="run only the headline workload at this batch (a small case for counter captures)")
    ap.add_argument("--profile-case", default=None, choices=["llama3_8b_gqa", "llama7b_layer_encode"],
                    help="run only this workload beside the headline (the GQA cache with 2 of its 32 layers), "
                         "a small case for counter captures")
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
