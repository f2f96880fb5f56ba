"""Seeded synthetic inputs shaped like the KV caches the GEAR pages evaluate on.

This module holds no part of the codec's arithmetic. It serves both sides of the
parity tests and the benchmark: the numpy functions produce any single (layer,
batch, head) unit on the CPU for the oracle, and the torch functions produce
whole tensors directly on the GPU. Both evaluate the same counter-based
generator, built only from exact integer operations, one float32 multiply and
one IEEE round-to-nearest conversion, so the two agree bit for bit.

Generator. Element number e of stream s under seed S draws 64 random bits from a
32-bit integer hash (Wellons' "lowbias32" construction, applied twice) and forms
the sum of four 16-bit uniforms (the Irwin-Hall approximation of a normal):
    N = (u1 + u2 + u3 + u4 - 131070) * c,   c = 1 / sqrt(4 * (65536^2 - 1) / 12)
which has mean 0, variance 1 and support |N| <= 3.47.

Small workloads whose description asks for i.i.d. N(0,1) entries (the tiny
single-head codec) instead draw true standard normals on the CPU from numpy's
seeded generator (PCG64, ``default_rng``), keyed by (seed, stream, layer, batch,
head) or (seed, stream, layer, step), and the torch side uploads those values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

_M32 = 0xFFFFFFFF
_C1 = 0x21F0AAAD
_C2 = 0x735A2D97
_NORM_C = np.float32(1.0 / math.sqrt(4.0 * (65536.0 ** 2 - 1.0) / 12.0))


# ---------------------------------------------------------------- numpy side
def _h32_np(x: np.ndarray) -> np.ndarray:
    x = x.astype(np.uint64) & _M32
    x ^= x >> np.uint64(16)
    x = (x * np.uint64(_C1)) & _M32
    x ^= x >> np.uint64(15)
    x = (x * np.uint64(_C2)) & _M32
    x ^= x >> np.uint64(15)
    return x


def _key(seed: int, stream: int) -> tuple[int, int, int]:
    k = [int(v) for v in _h32_np(np.array([seed & _M32, (seed >> 32) & _M32, stream & _M32],
                                          dtype=np.uint64))]
    return k[0] ^ k[2], int(_h32_np(np.array([k[1] ^ 0x9E3779B9], np.uint64))[0]), k[1]


def normal_np(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """float32 N(0,1)-like values at element indices idx (int64 array)."""
    k1, k2, k3 = _key(seed, stream)
    idx = idx.astype(np.uint64)
    lo = idx & np.uint64(_M32)
    hi = idx >> np.uint64(32)
    a = _h32_np(lo ^ np.uint64(k1) ^ _h32_np(hi ^ np.uint64(k3)))
    b = _h32_np(a ^ np.uint64(k2))
    s = (a & 0xFFFF) + (a >> np.uint64(16)) + (b & 0xFFFF) + (b >> np.uint64(16))
    return (s.astype(np.int64) - 131070).astype(np.float32) * _NORM_C


def uniform_u32_np(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    k1, k2, k3 = _key(seed, stream)
    idx = idx.astype(np.uint64)
    a = _h32_np((idx & np.uint64(_M32)) ^ np.uint64(k1) ^ _h32_np((idx >> np.uint64(32)) ^ np.uint64(k3)))
    return _h32_np(a ^ np.uint64(k2)).astype(np.uint32)


# ---------------------------------------------------------------- torch side
def _mul32_t(x, c: int):
    # (x * c) mod 2^32 with every partial product below 2^48 (no int64 overflow).
    lo, hi = c & 0xFFFF, c >> 16
    return (x * lo + (((x * hi) & 0xFFFF) << 16)) & _M32


def _h32_t(x):
    x = x & _M32
    x = x ^ (x >> 16)
    x = _mul32_t(x, _C1)
    x = x ^ (x >> 15)
    x = _mul32_t(x, _C2)
    x = x ^ (x >> 15)
    return x


def normal_torch(seed: int, stream: int, idx):
    """Same values as normal_np, for an int64 torch tensor of indices (any device)."""
    import torch
    k1, k2, k3 = _key(seed, stream)
    lo = idx & _M32
    hi = idx >> 32
    a = _h32_t(lo ^ k1 ^ _h32_t(hi ^ k3))
    b = _h32_t(a ^ k2)
    s = (a & 0xFFFF) + (a >> 16) + (b & 0xFFFF) + (b >> 16)
    return (s - 131070).to(torch.float32) * float(_NORM_C)


# ------------------------------------------------------- dtype conversion
def to_dtype_exact_np(x32: np.ndarray, dtype: str) -> np.ndarray:
    """Round float32 values to the cache dtype (round to nearest even) and return
    them as float32 holding the exact rounded values."""
    if dtype == "f32":
        return x32.astype(np.float32)
    if dtype == "f16":
        return x32.astype(np.float16).astype(np.float32)
    if dtype == "bf16":
        b = x32.astype(np.float32).view(np.uint32).astype(np.uint64)
        r = ((b + 0x7FFF + ((b >> 16) & 1)) >> 16) << 16
        return (r & _M32).astype(np.uint32).view(np.float32)
    raise ValueError(dtype)


def torch_dtype(dtype: str):
    import torch
    return {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}[dtype]


# ------------------------------------------------------------ workloads
@dataclass(frozen=True)
class Workload:
    """One synthetic workload. Sizes follow the pages' models (LLaMA-class heads,
    d = 128) and the stated codec settings."""
    name: str
    layers: int
    B: int
    H: int          # kv heads
    Hq: int         # query heads
    n: int          # compressed context per unit
    d: int
    dtype: str
    bits: int
    group: int
    s: float
    rank: int
    iters: int
    buffer_len: int
    buffer_fill: int    # tokens in the buffer at decode time
    buffer_rank: int
    seed: int
    k_channel_scale: bool   # K has per-(head, channel) log-uniform std in [0.5, 8]
    spike_frac: float       # fraction of K entries multiplied by 10 (tiny workload)
    cpu_normal: bool = False   # true N(0,1) draws from numpy's seeded generator (small workloads)


WORKLOADS = {
    # one 256 x 128 fp32 K matrix with 1% spiked entries, matching N(0,1) V and q
    "tiny": Workload("tiny", 1, 1, 1, 1, 256, 128, "f32", 4, 64, 0.02, 4, 3, 20, 0, 2,
                     1001, False, 0.01, cpu_normal=True),
    # LLaMA-7B-shaped layer: encode K and V of 32 heads x 4096 tokens, fp16
    "llama7b_layer_encode": Workload("llama7b_layer_encode", 1, 1, 32, 32, 4096, 128, "f16",
                                     4, 64, 0.02, 4, 3, 20, 0, 2, 1002, True, 0.0),
    # decode step: batch 16, 32 heads, 8192 compressed tokens + a full 20-token buffer
    "decode_b16_ctx8192": Workload("decode_b16_ctx8192", 1, 16, 32, 32, 8192, 128, "f16",
                                   4, 64, 0.02, 4, 3, 20, 20, 2, 1003, True, 0.0),
    # 2-bit codec at high batch: batch 64, 32 heads, 8192 tokens, r = 8, s = 5%
    "twobit_b64_ctx8192": Workload("twobit_b64_ctx8192", 1, 64, 32, 32, 8192, 128, "f16",
                                   2, 32, 0.05, 8, 3, 20, 0, 2, 1004, True, 0.0),
    # LLaMA-3-8B-shaped GQA cache: 32 layers, 8 kv heads, 32 query heads, bf16
    "llama3_8b_gqa": Workload("llama3_8b_gqa", 32, 8, 8, 32, 32768, 128, "bf16",
                              4, 64, 0.02, 4, 3, 20, 20, 2, 1005, True, 0.0),
}

# stream ids
S_K, S_V, S_Q, S_KBUF, S_VBUF, S_KNEW, S_VNEW, S_SPIKE = 1, 2, 3, 4, 5, 6, 7, 8


def channel_sigma(w: Workload, layer: int) -> np.ndarray:
    """float32 [H][d] per-(head, channel) std of K: exp(U(ln 0.5, ln 8))."""
    if not w.k_channel_scale:
        return np.ones((w.H, w.d), np.float32)
    u = uniform_u32_np(w.seed, 100 + layer, np.arange(w.H * w.d, dtype=np.int64))
    lo, hi = math.log(0.5), math.log(8.0)
    v = lo + (u.astype(np.float64) / 4294967296.0) * (hi - lo)
    return np.exp(v).astype(np.float32).reshape(w.H, w.d)


def spike_positions(w: Workload) -> np.ndarray:
    """Flat indices (within one unit) of the K entries multiplied by 10."""
    if w.spike_frac <= 0:
        return np.zeros(0, np.int64)
    total = w.n * w.d
    m = int(round(w.spike_frac * total))
    # seeded choice without replacement: order all entries by a hash, take the first m
    keys = uniform_u32_np(w.seed, S_SPIKE, np.arange(total, dtype=np.int64))
    return np.sort(np.argsort(keys, kind="stable")[:m]).astype(np.int64)


def _unit_index(w: Workload, layer: int, b: int, h: int, n: int) -> np.ndarray:
    base = ((layer * w.B + b) * w.H + h) * n * w.d
    return base + np.arange(n * w.d, dtype=np.int64)


def kv_unit_np(w: Workload, which: str, layer: int, b: int, h: int, n: int | None = None) -> np.ndarray:
    """float32 [n][d] exact (dtype-rounded) values of one unit of K or V."""
    n = w.n if n is None else n
    stream = S_K if which == "k" else S_V
    if w.cpu_normal:
        x = np.random.default_rng([w.seed, stream, layer, b, h]).standard_normal((n, w.d), dtype=np.float32)
    else:
        x = normal_np(w.seed, stream, _unit_index(w, layer, b, h, n)).reshape(n, w.d)
    if which == "k":
        x = x * channel_sigma(w, layer)[h][None, :]
        sp = spike_positions(w)
        sp = sp[sp < n * w.d]
        if sp.size:
            x.reshape(-1)[sp] *= np.float32(10.0)
    return to_dtype_exact_np(x, w.dtype)


def kv_tensor_torch(w: Workload, which: str, layer: int, device, n: int | None = None):
    """[B][H][n][d] tensor in the workload dtype, generated on `device` in chunks
    of whole units (bounded temporaries)."""
    import torch
    n = w.n if n is None else n
    if w.cpu_normal:
        x = np.stack([kv_unit_np(w, which, layer, b, h, n) for b in range(w.B) for h in range(w.H)])
        return torch.from_numpy(x.reshape(w.B, w.H, n, w.d)).to(device=device, dtype=torch_dtype(w.dtype))
    stream = S_K if which == "k" else S_V
    out = torch.empty((w.B * w.H, n, w.d), dtype=torch_dtype(w.dtype), device=device)
    sig = torch.from_numpy(channel_sigma(w, layer)).to(device) if which == "k" else None
    sp = spike_positions(w) if which == "k" else np.zeros(0, np.int64)
    sp = sp[sp < n * w.d]
    spt = torch.from_numpy(sp).to(device) if sp.size else None
    per_unit = n * w.d
    step = max(1, (1 << 26) // per_unit)
    base0 = layer * w.B * w.H * per_unit
    for u0 in range(0, w.B * w.H, step):
        u1 = min(w.B * w.H, u0 + step)
        idx = base0 + u0 * per_unit + torch.arange((u1 - u0) * per_unit, device=device, dtype=torch.int64)
        x = normal_torch(w.seed, stream, idx).view(u1 - u0, n, w.d)
        del idx
        if sig is not None:
            h = torch.arange(u0, u1, device=device) % w.H
            x.mul_(sig[h][:, None, :])
            if spt is not None:
                xs = x.view(u1 - u0, n * w.d)
                xs[:, spt] *= 10.0
        out[u0:u1] = x.to(out.dtype)
    return out.view(w.B, w.H, n, w.d)


def rows_np(w: Workload, stream: int, layer: int, step: int, heads: int) -> np.ndarray:
    """float32 [B][heads][d] exact values of a per-step row tensor (q, buffer or new token)."""
    if w.cpu_normal:
        x = np.random.default_rng([w.seed, stream, layer, step]).standard_normal((w.B, heads, w.d), dtype=np.float32)
        return to_dtype_exact_np(x, w.dtype)
    base = ((layer * 1_000_003 + step) * w.B * heads) * w.d
    idx = base + np.arange(w.B * heads * w.d, dtype=np.int64)
    return to_dtype_exact_np(normal_np(w.seed, stream, idx), w.dtype).reshape(w.B, heads, w.d)


def rows_torch(w: Workload, stream: int, layer: int, step: int, heads: int, device):
    import torch
    if w.cpu_normal:
        return torch.from_numpy(rows_np(w, stream, layer, step, heads)).to(device=device, dtype=torch_dtype(w.dtype))
    base = ((layer * 1_000_003 + step) * w.B * heads) * w.d
    idx = base + torch.arange(w.B * heads * w.d, device=device, dtype=torch.int64)
    return normal_torch(w.seed, stream, idx).view(w.B, heads, w.d).to(torch_dtype(w.dtype))
