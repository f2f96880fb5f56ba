"""CPU oracle of the GEAR KV-cache codec and the attention that consumes it.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The product path
(the CUDA library and its Python binding) never imports, links or runs it, and
it shares no code with them.

The arithmetic lives in ``gear_oracle.c`` (plain loops, one function per step
of the method, each citing the passage it follows). This module only marshals
numpy arrays into that library and holds the host-side bookkeeping of the
streaming buffer (GEAR: Efficient KV Cache Compression for LLM Inference,
Q3 "Streaming strategy").
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, field

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gear_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# Compiler flags: strict IEEE binary32/binary64, no contraction into FMA.
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(force: bool = False) -> str:
    """Compile gear_oracle.c into liboracle.so next to it (gcc)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", *CFLAGS, "-o", _LIB, _SRC, "-lm"])
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_LIB)
        P = ctypes.c_void_p
        i32 = ctypes.c_int32
        L.oracle_num_outliers.argtypes = [ctypes.c_float, i32]
        L.oracle_num_outliers.restype = i32
        L.oracle_select_outliers.argtypes = [P, i32, i32, P]
        L.oracle_quantize_token.argtypes = [P, i32, i32, i32, P, i32, i32, P, P, P, P, P]
        L.oracle_splitmix64_next.argtypes = [ctypes.POINTER(ctypes.c_uint64)]
        L.oracle_splitmix64_next.restype = ctypes.c_uint64
        L.oracle_start_matrix.argtypes = [ctypes.c_uint64, i32, i32, P]
        L.oracle_power_iteration.argtypes = [P, i32, i32, i32, i32, P, P, P]
        L.oracle_encode_unit.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, i32, ctypes.c_uint64,
                                         P, P, P, P, P, P, P, P]
        L.oracle_reconstruct_unit.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        L.oracle_attention.argtypes = [P, P, P, i32, i32, ctypes.c_double, P]
        L.oracle_quantize_channels.argtypes = [P, i32, i32, i32, i32, P, P, P, P, P]
        L.oracle_encode_unit_channels.argtypes = [P, i32, i32, i32, i32, i32, i32, i32, ctypes.c_uint64,
                                                  P, P, P, P, P, P, P, P]
        L.oracle_reconstruct_unit_channels.argtypes = [i32, i32, i32, i32, i32, i32, P, P, P, P, P, P, P, P]
        _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


# --------------------------------------------------------------------------
# Parameters (same meaning as the C ABI's gear_params).
# --------------------------------------------------------------------------
@dataclass
class Params:
    bits: int = 4
    group_size: int = 64
    outlier_frac: float = 0.02
    rank: int = 4
    power_iters: int = 3
    buffer_len: int = 20
    buffer_rank: int = 2
    seed: int = 0
    meta_f16: bool = False   # scale and zero stored as binary16 (byte-lean metadata)
    channel_groups: bool = False   # KIVI-combined keys: per-channel groups of group_size tokens


def num_outliers(s: float, d: int) -> int:
    return int(lib().oracle_num_outliers(ctypes.c_float(s), d))


def select_outliers(x: np.ndarray, k: int) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    idx = np.zeros(k, dtype=np.int32)
    lib().oracle_select_outliers(_p(x), x.shape[0], k, _p(idx))
    return idx


def quantize_token(x: np.ndarray, bits: int, g: int, oidx: np.ndarray, meta_f16: bool = False):
    """One token: returns (codes u32[W], scale f32[G], zero f32[G], dhat f32[d], resid f32[d])."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    d = x.shape[0]
    oidx = np.ascontiguousarray(oidx, dtype=np.int32)
    codes = np.zeros(d * bits // 32, dtype=np.uint32)
    scale = np.zeros(d // g, dtype=np.float32)
    zero = np.zeros(d // g, dtype=np.float32)
    dhat = np.zeros(d, dtype=np.float32)
    resid = np.zeros(d, dtype=np.float32)
    lib().oracle_quantize_token(_p(x), d, bits, g, _p(oidx), oidx.shape[0], int(meta_f16), _p(codes), _p(scale),
                                _p(zero), _p(dhat), _p(resid))
    return codes, scale, zero, dhat, resid


def splitmix64_stream(seed: int, count: int) -> list[int]:
    st = ctypes.c_uint64(seed)
    return [int(lib().oracle_splitmix64_next(ctypes.byref(st))) for _ in range(count)]


def start_matrix(seed: int, d: int, r: int) -> np.ndarray:
    q0 = np.zeros((d, r), dtype=np.float64)
    lib().oracle_start_matrix(ctypes.c_uint64(seed), d, r, _p(q0))
    return q0


def power_iteration(R: np.ndarray, r: int, T: int, q0: np.ndarray):
    R = np.ascontiguousarray(R, dtype=np.float32)
    n, d = R.shape
    q0 = np.ascontiguousarray(q0, dtype=np.float64)
    L = np.zeros((n, r), dtype=np.float64)
    Rf = np.zeros((d, r), dtype=np.float64)
    lib().oracle_power_iteration(_p(R), n, d, r, T, _p(q0), _p(L), _p(Rf))
    return L, Rf


@dataclass
class Unit:
    """Encoding of one (batch, head) matrix block of n tokens."""
    codes: np.ndarray   # u32 [n][W]
    scale: np.ndarray   # f32 [n][G]
    zero: np.ndarray    # f32 [n][G]
    oidx: np.ndarray    # i32 [n][k]
    oval: np.ndarray    # f32 [n][k]
    resid: np.ndarray   # f32 [n][d]
    L: np.ndarray       # f64 [n][r]
    Rf: np.ndarray      # f64 [d][r]
    rank: int = 0


def quantize_channels(X: np.ndarray, bits: int, g: int, is_out: np.ndarray):
    """Per-channel min-max quantization over groups of g consecutive tokens (the
    KIVI-combined key quantizer): returns (codes u32[n][W], scale f32[ng][d],
    zero f32[ng][d], resid f32[n][d])."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    n, d = X.shape
    ng = (n + g - 1) // g
    m = np.ascontiguousarray(is_out, dtype=np.int8)
    codes = np.zeros((n, d * bits // 32), np.uint32)
    scale = np.zeros((ng, d), np.float32)
    zero = np.zeros((ng, d), np.float32)
    resid = np.zeros((n, d), np.float32)
    lib().oracle_quantize_channels(_p(X), n, d, bits, g, _p(m), _p(codes), _p(scale), _p(zero), _p(resid))
    return codes, scale, zero, resid


def encode_unit(X: np.ndarray, p: Params, rank: int | None = None) -> Unit:
    """Steps 1-5 on one unit X [n][d] (float32 holding the exact input values).
    With p.channel_groups the quantizer is the KIVI-combined key quantizer and
    scale/zero are [ceil(n/g)][d]."""
    X = np.ascontiguousarray(X, dtype=np.float32)
    n, d = X.shape
    r = p.rank if rank is None else rank
    k = num_outliers(p.outlier_frac, d)
    if p.channel_groups:
        ng = (n + p.group_size - 1) // p.group_size
        u = Unit(codes=np.zeros((n, d * p.bits // 32), np.uint32), scale=np.zeros((ng, d), np.float32),
                 zero=np.zeros((ng, d), np.float32), oidx=np.zeros((n, k), np.int32),
                 oval=np.zeros((n, k), np.float32), resid=np.zeros((n, d), np.float32),
                 L=np.zeros((n, r), np.float64), Rf=np.zeros((d, r), np.float64), rank=r)
        lib().oracle_encode_unit_channels(_p(X), n, d, p.bits, p.group_size, k, r, p.power_iters,
                                          ctypes.c_uint64(p.seed), _p(u.codes), _p(u.scale), _p(u.zero),
                                          _p(u.oidx), _p(u.oval), _p(u.resid), _p(u.L), _p(u.Rf))
        return u
    W = d * p.bits // 32
    G = d // p.group_size
    u = Unit(codes=np.zeros((n, W), np.uint32), scale=np.zeros((n, G), np.float32),
             zero=np.zeros((n, G), np.float32), oidx=np.zeros((n, k), np.int32),
             oval=np.zeros((n, k), np.float32), resid=np.zeros((n, d), np.float32),
             L=np.zeros((n, r), np.float64), Rf=np.zeros((d, r), np.float64), rank=r)
    lib().oracle_encode_unit(_p(X), n, d, p.bits, p.group_size, k, int(p.meta_f16), r, p.power_iters,
                             ctypes.c_uint64(p.seed), _p(u.codes), _p(u.scale), _p(u.zero),
                             _p(u.oidx), _p(u.oval), _p(u.resid), _p(u.L), _p(u.Rf))
    return u


def reconstruct_unit(u: Unit, p: Params) -> np.ndarray:
    """Step 6: X_hat [n][d] (float64) of an encoded unit."""
    n = u.codes.shape[0]
    d = u.resid.shape[1]
    k = u.oidx.shape[1]
    Xh = np.zeros((n, d), dtype=np.float64)
    fn = lib().oracle_reconstruct_unit_channels if p.channel_groups else lib().oracle_reconstruct_unit
    fn(n, d, p.bits, p.group_size, k, u.rank, _p(u.codes), _p(u.scale), _p(u.zero), _p(u.oidx), _p(u.oval),
       _p(u.L), _p(u.Rf), _p(Xh))
    return Xh


def attention(q: np.ndarray, K: np.ndarray, V: np.ndarray, scale: float) -> np.ndarray:
    """Step 7: softmax(scale q.K^T) V for one query vector, float64."""
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    out = np.zeros(q.shape[0], dtype=np.float64)
    lib().oracle_attention(_p(q), _p(K), _p(V), K.shape[0], K.shape[1], float(scale), _p(out))
    return out


# --------------------------------------------------------------------------
# Host-side bookkeeping: a cache of blocks per unit plus the streaming buffer.
# --------------------------------------------------------------------------
def _map_units(fn, items, threads: int):
    if threads <= 1:
        return [fn(x) for x in items]
    # ctypes releases the GIL while the C oracle runs, so threads run in parallel.
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))


@dataclass
class Cache:
    """Oracle of one compressed tensor (K or V) of shape [B][H][*][d]."""
    p: Params
    B: int
    H: int
    d: int
    blocks: list = field(default_factory=list)    # list over blocks of list over units of Unit
    buffer: list = field(default_factory=list)    # list of float32 [B][H][d] rows

    @property
    def n_comp(self) -> int:
        return sum(b[0].codes.shape[0] for b in self.blocks)

    def encode(self, kv: np.ndarray, threads: int = 1) -> None:
        """Block 0 from a prefill tensor kv [B][H][n][d] (float32 exact values)."""
        assert not self.blocks and not self.buffer
        units = [kv[b, h] for b in range(self.B) for h in range(self.H)]
        self.blocks.append(_map_units(lambda X: encode_unit(X, self.p, self.p.rank), units, threads))

    def append(self, row: np.ndarray, threads: int = 1) -> None:
        """One new token per unit, row [B][H][d]. Flush first if the buffer is full."""
        if len(self.buffer) == self.p.buffer_len:
            blk = np.stack(self.buffer, axis=2)  # [B][H][n_b][d]
            units = [blk[b, h] for b in range(self.B) for h in range(self.H)]
            self.blocks.append(_map_units(lambda X: encode_unit(X, self.p, self.p.buffer_rank),
                                          units, threads))
            self.buffer = []
        self.buffer.append(np.array(row, dtype=np.float32))

    def dense(self) -> np.ndarray:
        """X_hat [B][H][n_comp + n_buf][d] float64: compressed blocks then buffer."""
        n = self.n_comp + len(self.buffer)
        out = np.zeros((self.B, self.H, n, self.d), dtype=np.float64)
        t0 = 0
        for blk in self.blocks:
            nb = blk[0].codes.shape[0]
            for u, unit in enumerate(blk):
                out[u // self.H, u % self.H, t0:t0 + nb] = reconstruct_unit(unit, self.p)
            t0 += nb
        for i, row in enumerate(self.buffer):
            out[:, :, t0 + i] = row
        return out


def decode_attn(kc: Cache, vc: Cache, q: np.ndarray, scale: float, prefill_len=None) -> np.ndarray:
    """Attention of q [B][Hq][d] over the reconstructed caches; float64 [B][Hq][d].
    Query head j reads kv-head j // (Hq // H).

    prefill_len (optional, B ints): batch row b's prefill was right-padded, so only
    the first prefill_len[b] tokens of block 0 are real (clamped to [0, block-0
    length]); the padding takes no part in the softmax, every later token does.
    A row with no real token gives 0. (Serving with prompts of different lengths;
    the paper decodes equal lengths, so this is a reading, not a passage.)"""
    B, Hq, d = q.shape
    H = kc.H
    Kd, Vd = kc.dense(), vc.dense()
    n = Kd.shape[2]
    n0 = kc.blocks[0][0].codes.shape[0] if kc.blocks else 0
    out = np.zeros((B, Hq, d), dtype=np.float64)
    for b in range(B):
        rows = np.arange(n)
        if prefill_len is not None:
            pl = min(max(int(prefill_len[b]), 0), n0)
            rows = rows[(rows < pl) | (rows >= n0)]
        if rows.size == 0:
            continue
        for j in range(Hq):
            h = j // (Hq // H)
            out[b, j] = attention(q[b, j], Kd[b, h][rows], Vd[b, h][rows], scale)
    return out
