"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare them."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import workloads as wl

TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


def oracle_params(p) -> oracle.Params:
    return oracle.Params(bits=p.bits, group_size=p.group_size, outlier_frac=p.outlier_frac, rank=p.rank,
                         power_iters=p.power_iters, buffer_len=p.buffer_len, buffer_rank=p.buffer_rank, seed=p.seed,
                         meta_f16=bool(p.meta_f16), channel_groups=bool(p.channel_groups))


def seeded_kv(seed: int, stream: int, shape, dtype: str, channel_scale: bool = False,
              dist: str = "irwin_hall") -> np.ndarray:
    """float32 array of exact dtype-rounded values from the shared generator, or
    (dist = "t3") heavy-tailed Student-t draws with 3 degrees of freedom from
    numpy's seeded generator, whose large entries exercise the outlier path."""
    n = int(np.prod(shape))
    if dist == "t3":
        x = np.random.default_rng([seed, stream]).standard_t(3, size=n).astype(np.float32).reshape(shape)
    else:
        x = wl.normal_np(seed, stream, np.arange(n, dtype=np.int64)).reshape(shape)
    if channel_scale:
        u = wl.uniform_u32_np(seed, 999, np.arange(shape[-1], dtype=np.int64))
        sig = np.exp(np.log(0.5) + (u / 4294967296.0) * (np.log(8.0) - np.log(0.5))).astype(np.float32)
        x = x * sig
    return wl.to_dtype_exact_np(x.astype(np.float32), dtype)


def to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(TORCH_DT[dtype]).cuda()


def unpack_codes(codes: np.ndarray, bits: int, d: int = 128) -> np.ndarray:
    c = np.arange(d)
    return (codes.view(np.uint32)[..., (c * bits) // 32] >> ((c * bits) % 32).astype(np.uint32)) & \
        np.uint32((1 << bits) - 1)


def gpu_block(cache, u: int, t0: int, t1: int, blk: int, rank: int):
    """Stored arrays of tokens [t0, t1) of unit u (numpy), L and Rf unscaled."""
    A = cache.arrays()
    n = t1 - t0
    e = 0
    while (2 << e) <= n:
        e += 1
    e //= 2
    L = A["lfac"][u, t0:t1, :rank].float().cpu().numpy().astype(np.float64) * 2.0 ** -e
    Rf = A["rfac"][u, blk, :, :rank].cpu().numpy().astype(np.float64) * 2.0 ** e   # [d][r]
    return {
        "codes": A["codes"][u, t0:t1].cpu().numpy(),
        "meta": A["meta"][u, t0:t1].cpu().numpy(),
        "oidx": A["oidx"][u, t0:t1].cpu().numpy(),
        "oval": A["oval"][u, t0:t1].float().cpu().numpy(),
        "L": L,
        "Rf": Rf,
    }


def compare_unit(g: dict, o: oracle.Unit, p, what: str = ""):
    """Bit-exact codes / scale / zero / outliers; tolerance on L Rf^T. Binary16
    metadata widens exactly to the oracle's binary32 copy of the stored values."""
    k = o.oidx.shape[1]
    meta = g["meta"].astype(np.float32)
    assert np.array_equal(g["codes"].view(np.uint32), o.codes), f"{what}: codes differ"
    assert np.array_equal(meta[..., 0].view(np.uint32), o.scale.view(np.uint32)), f"{what}: scale differs"
    assert np.array_equal(meta[..., 1].view(np.uint32), o.zero.view(np.uint32)), f"{what}: zero differs"
    if k:
        assert np.array_equal(g["oidx"][:, :k].astype(np.int32), o.oidx), f"{what}: outlier index differs"
        assert np.array_equal(g["oval"][:, :k].view(np.uint32), o.oval.view(np.uint32)), f"{what}: outlier value"
    if o.rank:
        lr_g = g["L"] @ g["Rf"].T
        lr_o = o.L @ o.Rf.T
        rmax = np.abs(o.resid).max()
        err = np.abs(lr_g - lr_o).max()
        assert err <= 1e-3 * rmax + 1e-30, f"{what}: L Rf^T error {err:.3e} > 1e-3 * max|R| = {1e-3 * rmax:.3e}"


def compare_dense(gd: np.ndarray, od: np.ndarray, scale: np.ndarray, g: int, what: str = ""):
    """|Xhat_gpu - Xhat_oracle| <= 1e-3 * (group scale) + tiny, elementwise."""
    sc = np.repeat(scale, g, axis=-1)
    err = np.abs(gd.astype(np.float64) - od)
    bound = 1e-3 * sc + 1e-6 * np.abs(od) + 1e-30
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} reconstructed entries off, worst {err[bad].max():.3e}"


def spread_units(U: int, count: int = 16) -> list[int]:
    """count unit indices spread evenly over [0, U), always with the first and the last."""
    if U <= count:
        return list(range(U))
    return sorted({round(i * (U - 1) / (count - 1)) for i in range(count)})


def pmap(fn, items, workers: int = 16):
    """fn over items on a thread pool (the oracle's C calls release the GIL)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    with ThreadPoolExecutor(max_workers=max(1, min(workers, os.cpu_count() or 1))) as ex:
        return list(ex.map(fn, items))
