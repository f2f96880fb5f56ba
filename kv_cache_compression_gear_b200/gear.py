"""ctypes binding of libgear (include/gear.h), with torch for memory and streams.

This module only marshals arguments: every step of the codec and of the
attention runs in the CUDA kernels of libgear.so. The C entry points are
re-exported under their own names (gear_encode, gear_decode_attn, ...); the
``Cache`` class wraps one compressed tensor whose device memory is a torch
uint8 buffer. Importing fails loudly if the library has not been built.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgear.so")

GEAR_OK, GEAR_ERR_INVALID_ARG, GEAR_ERR_UNSUPPORTED, GEAR_ERR_CAPACITY = 0, 1, 2, 3
GEAR_ERR_CUDA, GEAR_ERR_TIMEOUT, GEAR_ERR_WORKSPACE = 4, 5, 6
GEAR_F16, GEAR_BF16, GEAR_F32 = 0, 1, 2

_DT = {torch.float16: GEAR_F16, torch.bfloat16: GEAR_BF16, torch.float32: GEAR_F32}
_TORCH = {v: k for k, v in _DT.items()}


class GearParams(ctypes.Structure):
    _fields_ = [("bits", ctypes.c_int32), ("group_size", ctypes.c_int32), ("outlier_frac", ctypes.c_float),
                ("rank", ctypes.c_int32), ("power_iters", ctypes.c_int32), ("buffer_len", ctypes.c_int32),
                ("buffer_rank", ctypes.c_int32), ("meta_f16", ctypes.c_int32), ("channel_groups", ctypes.c_int32),
                ("seed", ctypes.c_uint64)]


class GearCacheStruct(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("d", ctypes.c_int32), ("n_max", ctypes.c_int32),
                ("nblk_max", ctypes.c_int32), ("dtype", ctypes.c_int32), ("p", GearParams),
                ("k", ctypes.c_int32), ("G", ctypes.c_int32), ("W", ctypes.c_int32), ("r_max", ctypes.c_int32),
                ("codes", ctypes.c_void_p), ("meta", ctypes.c_void_p), ("oidx", ctypes.c_void_p),
                ("oval", ctypes.c_void_p), ("lfac", ctypes.c_void_p), ("rfac", ctypes.c_void_p),
                ("buf", ctypes.c_void_p), ("n_comp", ctypes.c_int32), ("n_buf", ctypes.c_int32),
                ("n_blk", ctypes.c_int32), ("blk0_len", ctypes.c_int32), ("blk0_rank", ctypes.c_int32),
                ("reserved1", ctypes.c_int32), ("page_tokens", ctypes.c_int32), ("num_pages", ctypes.c_int32),
                ("pages_per_row", ctypes.c_int32), ("reserved2", ctypes.c_int32), ("table", ctypes.c_void_p),
                ("rows", ctypes.c_void_p), ("host", ctypes.c_void_p)]


class GearError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"libgear.so is not built ({LIB_PATH}); run __graft_entry__.build()")
    L = ctypes.CDLL(LIB_PATH)
    P, S = ctypes.c_void_p, ctypes.c_size_t
    i32 = ctypes.c_int32
    pp = ctypes.POINTER(GearParams)
    pc = ctypes.POINTER(GearCacheStruct)
    sig = {
        "gear_num_outliers": (i32, [ctypes.c_float, i32]),
        "gear_validate_params": (i32, [pp, i32]),
        "gear_cache_bytes": (S, [pp, i32, i32, i32, i32, i32, i32]),
        "gear_cache_init": (i32, [pc, pp, i32, i32, i32, i32, i32, i32, P, S]),
        "gear_cache_reset": (i32, [pc]),
        "gear_encode_workspace_bytes": (S, [pc, i32]),
        "gear_encode": (i32, [pc, P, i32, P, S, P]),
        "gear_encode_batch_workspace_bytes": (S, [i32, P, i32]),
        "gear_encode_batch": (i32, [i32, P, P, i32, P, S, P]),
        "gear_decode_workspace_bytes": (S, [pc, pc, i32]),
        "gear_decode_attn": (i32, [pc, pc, P, i32, ctypes.c_float, P, i32, P, S, P]),
        "gear_decode_attn_ragged": (i32, [pc, pc, P, i32, ctypes.c_float, P, i32, P, P, S, P]),
        "gear_decode_attn_noalloc": (i32, [pc, pc, P, i32, ctypes.c_float, P, i32, P]),
        "gear_append_workspace_bytes": (S, [pc]),
        "gear_append_buffer": (i32, [pc, pc, P, P, P, S, P]),
        "gear_decode_dense": (i32, [pc, P, P]),
        "gear_paged_host_ints": (S, [i32, i32, i32]),
        "gear_paged_cache_bytes": (S, [pp, i32, i32, i32, i32, i32, i32, i32, i32]),
        "gear_paged_cache_init": (i32, [pc, pp, i32, i32, i32, i32, i32, i32, i32, i32, P, S, P, S, P]),
        "gear_encode_rows_workspace_bytes": (S, [pc, i32, i32]),
        "gear_encode_rows": (i32, [pc, P, i32, P, i32, P, S, P]),
        "gear_append_rows_workspace_bytes": (S, [pc]),
        "gear_append_rows": (i32, [pc, pc, P, i32, P, P, P, S, P]),
        "gear_release_rows": (i32, [pc, P, i32, P]),
        "gear_get_device_status": (i32, [ctypes.POINTER(i32)]),
        "gear_selftest_wait_timeout": (i32, [ctypes.c_uint32, P]),
        "gear_status_string": (ctypes.c_char_p, [i32]),
        "gear_version": (ctypes.c_char_p, []),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    return L, list(sig)


lib, EXPORTS = _load()
for _name in EXPORTS:
    globals()[_name] = getattr(lib, _name)


def status_string(s: int) -> str:
    return lib.gear_status_string(s).decode()


def _check(status: int, what: str):
    if status != GEAR_OK:
        raise GearError(status, what)


def _stream_ptr(stream=None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, power_iters=3, buffer_len=20, buffer_rank=2,
                seed=0, meta_f16=False, channel_groups=False) -> GearParams:
    return GearParams(bits, group_size, outlier_frac, rank, power_iters, buffer_len, buffer_rank, int(meta_f16),
                      int(channel_groups), seed)


class _Workspace:
    """Grow-only device scratch buffer owned by torch."""

    def __init__(self):
        self.buf = None

    def get(self, nbytes: int, device) -> tuple[int, int]:
        if nbytes == 0:
            return 0, 0
        if self.buf is None or self.buf.numel() < nbytes or self.buf.device != torch.device(device):
            self.buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device)
        p = self.buf.data_ptr()
        p = (p + 255) & ~255
        return p, nbytes


_ws = _Workspace()


class Cache:
    """One compressed tensor (K or V) of shape [B][H][*][128] on a CUDA device."""

    def __init__(self, params: GearParams, B: int, H: int, n_max: int, nblk_max: int, dtype: torch.dtype,
                 device="cuda", d: int = 128):
        self.params = params
        self.dtype = dtype
        self.device = torch.device(device)
        nbytes = lib.gear_cache_bytes(ctypes.byref(params), B, H, d, n_max, nblk_max, _DT[dtype])
        if nbytes == 0:
            _check(lib.gear_validate_params(ctypes.byref(params), d) or GEAR_ERR_INVALID_ARG, "gear_cache_bytes")
        self.mem = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        base = (self.mem.data_ptr() + 255) & ~255
        self.c = GearCacheStruct()
        _check(lib.gear_cache_init(ctypes.byref(self.c), ctypes.byref(params), B, H, d, n_max, nblk_max, _DT[dtype],
                                   ctypes.c_void_p(base), nbytes), "gear_cache_init")

    # counters
    @property
    def n_comp(self) -> int:
        return self.c.n_comp

    @property
    def n_buf(self) -> int:
        return self.c.n_buf

    @property
    def n_blk(self) -> int:
        return self.c.n_blk

    def reset(self):
        """gear_cache_reset: empty the cache (host counters only) for a new encode."""
        _check(lib.gear_cache_reset(ctypes.byref(self.c)), "gear_cache_reset")

    def encode(self, kv: torch.Tensor, stream=None):
        assert kv.is_cuda and kv.dtype == self.dtype and kv.is_contiguous()
        B, H, n, d = kv.shape
        nbytes = lib.gear_encode_workspace_bytes(ctypes.byref(self.c), n)
        wp, wn = _ws.get(nbytes, kv.device)
        _check(lib.gear_encode(ctypes.byref(self.c), ctypes.c_void_p(kv.data_ptr()), n, ctypes.c_void_p(wp), wn,
                               _stream_ptr(stream)), "gear_encode")

    def dense(self, stream=None) -> torch.Tensor:
        c = self.c
        out = torch.empty((c.B, c.H, c.n_comp + c.n_buf, c.d), dtype=torch.float32, device=self.device)
        _check(lib.gear_decode_dense(ctypes.byref(c), ctypes.c_void_p(out.data_ptr()), _stream_ptr(stream)),
               "gear_decode_dense")
        return out

    # raw views of the stored arrays (for tests)
    def _view(self, ptr, count, dtype):
        off = ptr - self.mem.data_ptr()
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return self.mem[off:off + nbytes].view(dtype)

    def arrays(self) -> dict:
        c = self.c
        U = c.B * c.H
        n = c.n_max
        ld = torch.float32 if self.dtype == torch.float32 else torch.float16
        k = max(c.k, 1)
        rp = (c.r_max + 3) // 4 * 4
        return {
            "codes": self._view(c.codes, U * n * c.W, torch.int32).view(U, n, c.W),
            # per-channel key groups: [U][ceil(n_max / g) + 1 slots][d][2]
            "meta": (self._view(c.meta, U * (-(-n // c.p.group_size) + 1) * c.d * 2, torch.float32)
                     .view(U, -1, c.d, 2) if c.p.channel_groups else
                     self._view(c.meta, U * n * c.G * 2, torch.float16 if c.p.meta_f16 else torch.float32)
                     .view(U, n, c.G, 2)),
            "oidx": self._view(c.oidx, U * n * k, torch.uint8).view(U, n, k),
            "oval": self._view(c.oval, U * n * k, self.dtype).view(U, n, k),
            "lfac": self._view(c.lfac, U * n * c.r_max, ld).view(U, n, c.r_max),
            "rfac": self._view(c.rfac, U * c.nblk_max * c.d * rp, torch.float32).view(U, c.nblk_max, c.d, rp),
            "buf": self._view(c.buf, U * c.p.buffer_len * c.d, self.dtype).view(U, c.p.buffer_len, c.d),
        }


def _rows_arg(rows):
    """Host int32 array of row indices (kept alive by the caller's reference)."""
    import numpy as np
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int32).reshape(-1))
    return r, ctypes.c_void_p(r.ctypes.data), int(r.size)


class PagedCache:
    """One compressed tensor in the paged layout: B rows (sequences) of H kv heads
    whose compressed tokens live in a pool of num_pages pages of page_tokens tokens.
    The host state (per-row counters, block-table mirror, free pages) is a numpy
    int32 array this object owns."""

    def __init__(self, params: GearParams, B: int, H: int, page_tokens: int, num_pages: int, pages_per_row: int,
                 nblk_max: int, dtype: torch.dtype, device="cuda", d: int = 128, stream=None):
        import numpy as np
        self.params = params
        self.dtype = dtype
        self.device = torch.device(device)
        nbytes = lib.gear_paged_cache_bytes(ctypes.byref(params), B, H, d, page_tokens, num_pages, pages_per_row,
                                            nblk_max, _DT[dtype])
        if nbytes == 0:
            raise GearError(GEAR_ERR_INVALID_ARG, "gear_paged_cache_bytes")
        nh = lib.gear_paged_host_ints(B, pages_per_row, num_pages)
        self.host = np.zeros(nh, dtype=np.int32)
        self.mem = torch.empty(nbytes + 256, dtype=torch.uint8, device=self.device)
        base = (self.mem.data_ptr() + 255) & ~255
        self.c = GearCacheStruct()
        _check(lib.gear_paged_cache_init(ctypes.byref(self.c), ctypes.byref(params), B, H, d, page_tokens, num_pages,
                                         pages_per_row, nblk_max, _DT[dtype], ctypes.c_void_p(base), nbytes,
                                         ctypes.c_void_p(self.host.ctypes.data), nh, _stream_ptr(stream)),
               "gear_paged_cache_init")

    @property
    def n_comp(self) -> int:
        return self.c.n_comp

    @property
    def n_buf(self) -> int:
        return self.c.n_buf

    def counters(self):
        """Copies of the per-row (block-0 length, blocks, buffer fill) and the table mirror."""
        B, ppr = self.c.B, self.c.pages_per_row
        h = self.host
        return h[:B].copy(), h[B:2 * B].copy(), h[2 * B:3 * B].copy(), h[3 * B:3 * B + B * ppr].reshape(B, ppr).copy()

    def free_pages(self) -> int:
        return int(self.host[-1])

    def encode_rows(self, rows, kv: torch.Tensor, stream=None):
        """gear_encode_rows: kv [len(rows)][H][n][d] becomes block 0 of the (empty) rows."""
        assert kv.is_cuda and kv.dtype == self.dtype and kv.is_contiguous()
        r, rp, nr = _rows_arg(rows)
        n = kv.shape[2]
        nbytes = lib.gear_encode_rows_workspace_bytes(ctypes.byref(self.c), nr, n)
        wp, wn = _ws.get(nbytes, kv.device)
        _check(lib.gear_encode_rows(ctypes.byref(self.c), rp, nr, ctypes.c_void_p(kv.data_ptr()), n,
                                    ctypes.c_void_p(wp), wn, _stream_ptr(stream)), "gear_encode_rows")

    def release_rows(self, rows, stream=None):
        r, rp, nr = _rows_arg(rows)
        _check(lib.gear_release_rows(ctypes.byref(self.c), rp, nr, _stream_ptr(stream)), "gear_release_rows")

    def _view(self, ptr, count, dtype):
        off = ptr - self.mem.data_ptr()
        nbytes = count * torch.empty((), dtype=dtype).element_size()
        return self.mem[off:off + nbytes].view(dtype)

    def arrays(self) -> dict:
        """Raw views: pool arrays [num_pages][H][P][...], rfac [U][nblk_max][d][r_pad], buf, table, rows."""
        c = self.c
        U = c.B * c.H
        NP, H, P = c.num_pages, c.H, c.page_tokens
        R = NP * H * P
        ld = torch.float32 if self.dtype == torch.float32 else torch.float16
        k = max(c.k, 1)
        rp = (c.r_max + 3) // 4 * 4
        return {
            "codes": self._view(c.codes, R * c.W, torch.int32).view(NP, H, P, c.W),
            # per-channel key groups: per unit [U][ceil(P * pages_per_row / g) + 1 slots][d][2]
            "meta": (self._view(c.meta, U * (-(-(P * c.pages_per_row) // c.p.group_size) + 1) * c.d * 2,
                                torch.float32).view(c.B, H, -1, c.d, 2) if c.p.channel_groups else
                     self._view(c.meta, R * c.G * 2, torch.float16 if c.p.meta_f16 else torch.float32)
                     .view(NP, H, P, c.G, 2)),
            "oidx": self._view(c.oidx, R * k, torch.uint8).view(NP, H, P, k),
            "oval": self._view(c.oval, R * k, self.dtype).view(NP, H, P, k),
            "lfac": self._view(c.lfac, R * c.r_max, ld).view(NP, H, P, c.r_max),
            "rfac": self._view(c.rfac, U * c.nblk_max * c.d * rp, torch.float32).view(c.B, H, c.nblk_max, c.d, rp),
            "buf": self._view(c.buf, U * c.p.buffer_len * c.d, self.dtype).view(c.B, H, c.p.buffer_len, c.d),
            "table": self._view(c.table, c.B * c.pages_per_row, torch.int32).view(c.B, c.pages_per_row),
            "rows": self._view(c.rows, 3 * c.B, torch.int32).view(3, c.B),
        }


def append_rows(kc: PagedCache, vc: PagedCache, rows, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
    """gear_append_rows: one token per listed row, k_new/v_new [len(rows)][H][d]."""
    assert k_new.is_cuda and k_new.dtype == kc.dtype and k_new.is_contiguous() and v_new.is_contiguous()
    r, rp, nr = _rows_arg(rows)
    nbytes = lib.gear_append_rows_workspace_bytes(ctypes.byref(kc.c))
    wp, wn = _ws.get(nbytes, k_new.device)
    _check(lib.gear_append_rows(ctypes.byref(kc.c), ctypes.byref(vc.c), rp, nr, ctypes.c_void_p(k_new.data_ptr()),
                                ctypes.c_void_p(v_new.data_ptr()), ctypes.c_void_p(wp), wn, _stream_ptr(stream)),
           "gear_append_rows")


def encode_batch(caches, kvs, stream=None):
    """gear_encode_batch: encodes kvs[i] [B][H][n][d] into caches[i] in shared launches."""
    assert len(caches) == len(kvs) and len(caches) > 0
    for c, kv in zip(caches, kvs):
        assert kv.is_cuda and kv.dtype == c.dtype and kv.is_contiguous()
    n = kvs[0].shape[2]
    cnt = len(caches)
    cptrs = (ctypes.c_void_p * cnt)(*[ctypes.addressof(c.c) for c in caches])
    xptrs = (ctypes.c_void_p * cnt)(*[kv.data_ptr() for kv in kvs])
    nbytes = lib.gear_encode_batch_workspace_bytes(cnt, cptrs, n)
    wp, wn = _ws.get(nbytes, kvs[0].device)
    _check(lib.gear_encode_batch(cnt, cptrs, xptrs, n, ctypes.c_void_p(wp), wn, _stream_ptr(stream)),
           "gear_encode_batch")


def decode_attn(kc: Cache, vc: Cache, q: torch.Tensor, softmax_scale: float, out_dtype=None, out=None,
                stream=None, prefill_len: torch.Tensor | None = None) -> torch.Tensor:
    """gear_decode_attn, or gear_decode_attn_ragged when prefill_len (int32 [B] on the
    device: real tokens at the head of each batch row's prefill) is given."""
    assert q.is_cuda and q.dtype == kc.dtype and q.is_contiguous()
    B, Hq, d = q.shape
    od = out_dtype or kc.dtype
    if out is None:
        out = torch.empty((B, Hq, d), dtype=od, device=q.device)
    nbytes = lib.gear_decode_workspace_bytes(ctypes.byref(kc.c), ctypes.byref(vc.c), Hq)
    if nbytes == 0:
        raise GearError(GEAR_ERR_INVALID_ARG, "gear_decode_workspace_bytes")
    wp, wn = _ws.get(nbytes, q.device)
    if prefill_len is not None:
        assert prefill_len.is_cuda and prefill_len.dtype == torch.int32 and prefill_len.is_contiguous()
        assert prefill_len.numel() == B
        _check(lib.gear_decode_attn_ragged(ctypes.byref(kc.c), ctypes.byref(vc.c), ctypes.c_void_p(q.data_ptr()),
                                           Hq, ctypes.c_float(softmax_scale), ctypes.c_void_p(out.data_ptr()),
                                           _DT[od], ctypes.c_void_p(prefill_len.data_ptr()), ctypes.c_void_p(wp),
                                           wn, _stream_ptr(stream)), "gear_decode_attn_ragged")
        return out
    _check(lib.gear_decode_attn(ctypes.byref(kc.c), ctypes.byref(vc.c), ctypes.c_void_p(q.data_ptr()), Hq,
                                ctypes.c_float(softmax_scale), ctypes.c_void_p(out.data_ptr()), _DT[od],
                                ctypes.c_void_p(wp), wn, _stream_ptr(stream)), "gear_decode_attn")
    return out


def append_buffer(kc: Cache, vc: Cache, k_new: torch.Tensor, v_new: torch.Tensor, stream=None):
    assert k_new.is_cuda and k_new.dtype == kc.dtype and k_new.is_contiguous() and v_new.is_contiguous()
    nbytes = lib.gear_append_workspace_bytes(ctypes.byref(kc.c))
    wp, wn = _ws.get(nbytes, k_new.device)
    _check(lib.gear_append_buffer(ctypes.byref(kc.c), ctypes.byref(vc.c), ctypes.c_void_p(k_new.data_ptr()),
                                  ctypes.c_void_p(v_new.data_ptr()), ctypes.c_void_p(wp), wn, _stream_ptr(stream)),
           "gear_append_buffer")


def device_status() -> int:
    v = ctypes.c_int32(0)
    _check(lib.gear_get_device_status(ctypes.byref(v)), "gear_get_device_status")
    return v.value
