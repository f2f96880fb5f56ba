"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs. Codes, scales, zero points and outliers are compared bit for
bit; the low-rank term, the reconstruction and attention within stated
tolerances (see gpu_helpers)."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.gpu_helpers import (TORCH_DT, compare_dense, compare_unit, gpu_block, oracle_params, pmap, seeded_kv,
                               spread_units, to_dev)

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_compression_gear_b200 as gear
else:
    gear = None


def _tol_out(dtype: str) -> float:
    return 8e-3 if dtype == "bf16" else 1e-3


def _encode_both(x: np.ndarray, dtype: str, p, n_max=None, nblk_max=4):
    B, H, n, d = x.shape
    kc = gear.Cache(p, B, H, n_max or n, nblk_max, TORCH_DT[dtype])
    kc.encode(to_dev(x, dtype))
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    op = oracle_params(p)
    units = [oracle.encode_unit(x[b, h], op) for b in range(B) for h in range(H)]
    return kc, units, op


# ------------------------------------------------------------------ encode
ENC_CASES = [
    # dtype, B, H, n, bits, g, s, r, T
    ("f16", 1, 2, 1, 4, 64, 0.02, 1, 3),
    ("f16", 1, 2, 2, 4, 64, 0.02, 2, 3),
    ("f16", 2, 1, 7, 4, 64, 0.02, 4, 3),
    ("f16", 1, 3, 33, 2, 32, 0.05, 4, 2),
    ("f16", 1, 2, 128, 4, 64, 0.02, 4, 3),
    ("f16", 1, 2, 129, 8, 64, 0.02, 4, 3),
    ("f16", 2, 2, 300, 4, 32, 0.02, 8, 3),
    ("f16", 1, 3, 1000, 4, 128, 0.02, 4, 3),
    ("f16", 1, 2, 257, 4, 64, 0.0, 0, 1),
    ("f16", 2, 2, 300, 4, 64, 0.0, 4, 3),    # GEAR-L: no outliers, low rank
    ("f16", 1, 2, 257, 4, 64, 0.1, 16, 2),
    ("bf16", 1, 2, 300, 4, 64, 0.02, 4, 3),
    ("bf16", 2, 2, 77, 2, 64, 0.05, 2, 1),
    ("f32", 1, 1, 256, 4, 64, 0.02, 4, 3),
    ("f32", 1, 2, 130, 8, 32, 0.05, 3, 2),
]

# heavy-tailed (Student-t, 3 degrees of freedom) inputs: large isolated entries
HEAVY_ENC_CASES = [
    # dtype, B, H, n, bits, g, s, r, T
    ("f16", 1, 2, 300, 4, 64, 0.02, 4, 3),
    ("bf16", 2, 1, 257, 2, 32, 0.05, 8, 3),
    ("f32", 1, 2, 130, 4, 128, 0.1, 4, 2),
]


# binary16 metadata (fp16 caches): 16-, 8- and 4-byte meta rows, GEAR-L
F16_META_ENC_CASES = [
    # B, H, n, bits, g, s, r, T
    (1, 2, 300, 4, 32, 0.02, 4, 3),
    (2, 2, 129, 4, 64, 0.02, 4, 3),
    (1, 3, 257, 2, 128, 0.05, 2, 2),
    (1, 2, 200, 8, 64, 0.0, 4, 3),
    (1, 2, 33, 4, 64, 0.1, 16, 2),
]


@pytest.mark.parametrize("dtype,B,H,n,bits,g,s,r,T", ENC_CASES)
def test_encode_matches_oracle(dtype, B, H, n, bits, g, s, r, T):
    _encode_case(dtype, B, H, n, bits, g, s, r, T, meta_f16=False)


@pytest.mark.parametrize("B,H,n,bits,g,s,r,T", F16_META_ENC_CASES)
def test_encode_f16_metadata_matches_oracle(B, H, n, bits, g, s, r, T):
    _encode_case("f16", B, H, n, bits, g, s, r, T, meta_f16=True)


@pytest.mark.parametrize("dtype,B,H,n,bits,g,s,r,T", HEAVY_ENC_CASES)
def test_encode_heavy_tailed_matches_oracle(dtype, B, H, n, bits, g, s, r, T):
    _encode_case(dtype, B, H, n, bits, g, s, r, T, meta_f16=False, dist="t3")


def _encode_case(dtype, B, H, n, bits, g, s, r, T, meta_f16, dist="irwin_hall"):
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, power_iters=T, seed=1234 + n,
                         meta_f16=meta_f16)
    x = seeded_kv(7 + n + bits, 1, (B, H, n, 128), dtype, channel_scale=True, dist=dist)
    kc, units, op = _encode_both(x, dtype, p)
    dense = kc.dense().cpu().numpy()
    for u, o in enumerate(units):
        gb = gpu_block(kc, u, 0, n, 0, r)
        compare_unit(gb, o, p, f"unit {u}")
        compare_dense(dense[u // H, u % H], oracle.reconstruct_unit(o, op), o.scale, g, f"unit {u}")


def test_encode_ties_and_constant_groups():
    # many exact ties in |x| (integers), constant groups, signed zeros
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.05, rank=4, seed=3)
    rng = np.random.default_rng(5)
    x = rng.integers(-4, 5, size=(1, 2, 200, 128)).astype(np.float32)
    x[0, 0, 3, :64] = 2.0
    x[0, 0, 4, :] = 0.0
    x[0, 1, 5, ::2] = -0.0
    kc, units, op = _encode_both(x, "f16", p)
    for u, o in enumerate(units):
        compare_unit(gpu_block(kc, u, 0, 200, 0, 4), o, p, f"unit {u}")


def test_encode_rank_deficient_residual():
    # (a) 8-bit codes with a group range of exactly 255: scale 1, every entry is
    # reproduced, the residual is zero and all factors must be zero
    p = gear.make_params(bits=8, group_size=64, outlier_frac=0.0, rank=4, seed=9)
    rng = np.random.default_rng(2)
    x = rng.integers(0, 256, size=(1, 1, 64, 128)).astype(np.float32)
    x[..., 0::64] = 0.0
    x[..., 1::64] = 255.0
    kc, units, op = _encode_both(x, "f16", p)
    g = gpu_block(kc, 0, 0, 64, 0, 4)
    compare_unit(g, units[0], p)
    assert not units[0].resid.any()
    assert not g["L"].any() and not g["Rf"].any()
    # (b) identical rows: the residual has rank 1, so three of four columns drop
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, seed=9)
    x = np.tile(seeded_kv(4, 1, (1, 128), "f16"), (1, 1, 64, 1))
    kc, units, op = _encode_both(x, "f16", p)
    g = gpu_block(kc, 0, 0, 64, 0, 4)
    compare_unit(g, units[0], p)
    R = units[0].resid.astype(np.float64)
    assert np.abs(g["L"] @ g["Rf"].T - R).max() <= 1e-3 * np.abs(R).max()


# ------------------------------------------------------------ decode + append
def _build_caches(dtype, B, H, n0, p, nappend, seed, n_max=None, nblk_max=None, dist="irwin_hall"):
    xk = seeded_kv(seed, 1, (B, H, n0, 128), dtype, channel_scale=True, dist=dist)
    xv = seeded_kv(seed, 2, (B, H, n0, 128), dtype, dist=dist)
    n_max = n_max or n0 + nappend + 1
    nblk_max = nblk_max or 2 + nappend // p.buffer_len
    kc = gear.Cache(p, B, H, n_max, nblk_max, TORCH_DT[dtype])
    vc = gear.Cache(p, B, H, n_max, nblk_max, TORCH_DT[dtype])
    op = oracle_params(p)
    ok, ov = oracle.Cache(op, B, H, 128), oracle.Cache(op, B, H, 128)
    if n0:
        kc.encode(to_dev(xk, dtype))
        vc.encode(to_dev(xv, dtype))
        ok.encode(xk)
        ov.encode(xv)
    for i in range(nappend):
        rk = seeded_kv(seed + 100 + i, 3, (B, H, 128), dtype)
        rv = seeded_kv(seed + 100 + i, 4, (B, H, 128), dtype)
        gear.append_buffer(kc, vc, to_dev(rk, dtype), to_dev(rv, dtype))
        ok.append(rk)
        ov.append(rv)
    torch.cuda.synchronize()
    return kc, vc, ok, ov


DEC_CASES = [
    # dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf
    ("f16", 2, 2, 2, 300, 0, 4, 64, 0.02, 4, 20, 2),
    ("f16", 1, 2, 8, 200, 5, 4, 64, 0.02, 4, 20, 2),
    ("f16", 2, 1, 4, 130, 45, 2, 32, 0.05, 8, 20, 2),
    ("f16", 1, 2, 2, 0, 7, 4, 64, 0.02, 4, 3, 1),
    ("f16", 1, 2, 2, 1000, 21, 4, 128, 0.0, 0, 20, 0),
    ("f16", 2, 2, 8, 300, 25, 4, 64, 0.0, 4, 20, 2),    # GEAR-L
    ("bf16", 1, 2, 2, 200, 3, 2, 32, 0.0, 8, 20, 2),    # GEAR-L
    ("bf16", 1, 2, 8, 257, 20, 4, 64, 0.02, 4, 20, 2),
    ("f32", 1, 1, 1, 256, 0, 4, 64, 0.02, 4, 20, 2),
    ("f32", 1, 2, 4, 64, 9, 8, 32, 0.05, 2, 4, 2),
    # eight query heads per kv head (the HQ = 8 decoder)
    ("f16", 1, 1, 8, 300, 5, 4, 64, 0.02, 4, 20, 2),
    ("f16", 2, 2, 16, 130, 45, 2, 32, 0.05, 8, 20, 2),
    ("bf16", 2, 2, 16, 200, 21, 4, 64, 0.0, 4, 20, 2),   # GEAR-L
    ("f32", 1, 1, 8, 150, 3, 4, 32, 0.02, 4, 20, 2),
]

# heavy-tailed inputs through encode, append and decode
HEAVY_DEC_CASES = [
    ("f16", 2, 2, 4, 300, 25, 4, 64, 0.02, 4, 20, 2),
    ("bf16", 1, 2, 16, 257, 3, 2, 32, 0.05, 8, 20, 2),
]


F16_META_DEC_CASES = [
    # B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf
    (2, 2, 2, 300, 25, 4, 32, 0.02, 4, 20, 2),
    (1, 2, 8, 257, 20, 4, 64, 0.02, 4, 20, 2),
    (1, 2, 4, 130, 45, 2, 128, 0.05, 8, 20, 2),
    (2, 2, 2, 300, 0, 8, 64, 0.0, 4, 20, 2),
    (1, 1, 8, 257, 20, 4, 64, 0.02, 4, 20, 2),
]


@pytest.mark.parametrize("dtype,B,H,Hq,n0,nappend,bits,g,s,r,n_b,r_buf", DEC_CASES)
def test_decode_and_append_match_oracle(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf):
    _decode_case(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, meta_f16=False)


@pytest.mark.parametrize("B,H,Hq,n0,nappend,bits,g,s,r,n_b,r_buf", F16_META_DEC_CASES)
def test_decode_f16_metadata_match_oracle(B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf):
    _decode_case("f16", B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, meta_f16=True)


@pytest.mark.parametrize("dtype,B,H,Hq,n0,nappend,bits,g,s,r,n_b,r_buf", HEAVY_DEC_CASES)
def test_decode_heavy_tailed_matches_oracle(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf):
    _decode_case(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, meta_f16=False, dist="t3")


def _decode_case(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, meta_f16, dist="irwin_hall"):
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, buffer_len=n_b, buffer_rank=r_buf,
                         power_iters=3, seed=77, meta_f16=meta_f16)
    kc, vc, ok, ov = _build_caches(dtype, B, H, n0, p, nappend, seed=11 + n0, dist=dist)
    assert kc.n_comp == ok.n_comp and kc.n_buf == len(ok.buffer) and kc.n_blk == len(ok.blocks)
    q = seeded_kv(99 + n0, 5, (B, Hq, 128), dtype)
    tau = 1.0 / math.sqrt(128)
    od = oracle.decode_attn(ok, ov, q, tau)
    vmax = np.abs(ov.dense()).max()
    for out_dt in [TORCH_DT[dtype], torch.float32]:
        out = gear.decode_attn(kc, vc, to_dev(q, dtype), tau, out_dtype=out_dt).float().cpu().numpy()
        err = np.abs(out - od).max()
        assert err <= _tol_out(dtype) * vmax, f"attention error {err:.3e} vs {_tol_out(dtype) * vmax:.3e}"
    # flushed blocks equal the oracle's blocks
    t0 = ok.blocks[0][0].codes.shape[0] if n0 else 0
    for bi, blk in enumerate(ok.blocks):
        if n0 and bi == 0:
            continue
        for u, o in enumerate(blk):
            compare_unit(gpu_block(kc, u, t0, t0 + n_b, bi, r_buf), o, p, f"K block {bi} unit {u}")
        t0 += n_b
    assert gear.device_status() == 0


RAGGED_CASES = [
    # dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, prefill lengths
    ("f16", 4, 2, 4, 300, 25, 4, 64, 0.02, 4, 20, 2, [0, 1, 157, 300]),
    ("bf16", 3, 2, 2, 257, 0, 4, 32, 0.05, 4, 20, 2, [0, 100, 400]),   # row 0: nothing real, output 0
    ("f32", 2, 1, 1, 64, 9, 8, 64, 0.02, 2, 4, 1, [33, 5]),
    ("f16", 2, 2, 8, 130, 21, 2, 128, 0.0, 4, 20, 2, [129, 31]),         # GEAR-L, GQA
    ("f16", 3, 1, 8, 200, 3, 4, 64, 0.02, 4, 20, 2, [0, 77, 200]),       # eight query heads per kv head
]


@pytest.mark.parametrize("dtype,B,H,Hq,n0,nappend,bits,g,s,r,n_b,r_buf,plen", RAGGED_CASES)
def test_ragged_prefill_decode_matches_oracle(dtype, B, H, Hq, n0, nappend, bits, g, s, r, n_b, r_buf, plen):
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, buffer_len=n_b, buffer_rank=r_buf,
                         power_iters=3, seed=41)
    kc, vc, ok, ov = _build_caches(dtype, B, H, n0, p, nappend, seed=5 + n0)
    q = seeded_kv(77 + n0, 5, (B, Hq, 128), dtype)
    tau = 1.0 / math.sqrt(128)
    od = oracle.decode_attn(ok, ov, q, tau, prefill_len=plen)
    vmax = np.abs(ov.dense()).max()
    pl = torch.tensor(plen, dtype=torch.int32, device="cuda")
    out = gear.decode_attn(kc, vc, to_dev(q, dtype), tau, out_dtype=torch.float32, prefill_len=pl).cpu().numpy()
    err = np.abs(out - od).max()
    assert err <= _tol_out(dtype) * vmax, f"attention error {err:.3e} vs {_tol_out(dtype) * vmax:.3e}"
    for b, n in enumerate(plen):
        if n <= 0 and nappend == 0:
            assert not out[b].any()
    assert gear.device_status() == 0


# ------------------------------------------------------------ batched encode
BATCH_CASES = [
    # dtype, count, B, H, n, bits, g, s, r, T
    ("f16", 2, 2, 2, 300, 4, 64, 0.02, 4, 3),
    ("bf16", 3, 1, 3, 129, 2, 32, 0.05, 8, 2),
    ("f32", 2, 1, 2, 200, 8, 128, 0.02, 3, 3),
    ("f16", 17, 1, 1, 65, 4, 64, 0.02, 2, 3),   # more than one launch
]


@pytest.mark.parametrize("dtype,count,B,H,n,bits,g,s,r,T", BATCH_CASES)
def test_encode_batch_matches_single_and_oracle(dtype, count, B, H, n, bits, g, s, r, T):
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, power_iters=T, seed=99 + n)
    op = oracle_params(p)
    xs = [seeded_kv(300 + i, 1, (B, H, n, 128), dtype, channel_scale=True) for i in range(count)]
    caches = [gear.Cache(p, B, H, n + 32, 2, TORCH_DT[dtype]) for _ in range(count)]
    gear.encode_batch(caches, [to_dev(x, dtype) for x in xs])
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    for i in sorted({0, count // 2, count - 1}):
        single = gear.Cache(p, B, H, n + 32, 2, TORCH_DT[dtype])
        single.encode(to_dev(xs[i], dtype))
        A, S = caches[i].arrays(), single.arrays()
        for name in ["codes", "meta", "oidx", "oval"]:
            assert torch.equal(A[name][:, :n], S[name][:, :n]), (i, name)
        assert caches[i].c.n_comp == n and caches[i].c.n_blk == 1
        dense = caches[i].dense().cpu().numpy()
        for u in range(B * H):
            o = oracle.encode_unit(xs[i][u // H, u % H], op)
            compare_unit(gpu_block(caches[i], u, 0, n, 0, r), o, p, f"tensor {i} unit {u}")
            compare_dense(dense[u // H, u % H], oracle.reconstruct_unit(o, op), o.scale, g, f"tensor {i} unit {u}")


# ------------------------------------------------------ full-size workloads
def _wparams(w: wl.Workload):
    return gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank, power_iters=w.iters,
                            buffer_len=w.buffer_len, buffer_rank=w.buffer_rank, seed=w.seed)


def _check_sampled_units(w, caches, units, op, p, layer=0, what=""):
    """Bit-exact encode of each sampled (b, h) unit of K and V against the oracle."""
    jobs = [(which, b, h) for which in ("k", "v") for (b, h) in units]
    refs = pmap(lambda j: oracle.encode_unit(wl.kv_unit_np(w, j[0], layer, j[1], j[2]), op), jobs)
    for (which, b, h), o in zip(jobs, refs):
        compare_unit(gpu_block(caches[which], b * w.H + h, 0, w.n, 0, w.rank), o, p, f"{what} {which} ({b},{h})")


def _workload_encode_check(w: wl.Workload, units_to_check, layer=0, n_extra=64, nblk=4):
    p = _wparams(w)
    op = oracle_params(p)
    caches = {}
    for which in ["k", "v"]:
        x = wl.kv_tensor_torch(w, which, layer, "cuda")
        c = gear.Cache(p, w.B, w.H, w.n + n_extra, nblk, TORCH_DT[w.dtype])
        c.encode(x)
        torch.cuda.synchronize()
        del x
        caches[which] = c
    assert gear.device_status() == 0
    _check_sampled_units(w, caches, units_to_check, op, p, layer, w.name)
    return p, caches


def _units_bh(w, count=16):
    return [(u // w.H, u % w.H) for u in spread_units(w.B * w.H, count)]


def test_full_tiny_workload():
    """The tiny single-head codec exactly as specified: fp32, true N(0,1) entries with
    1 % of K spiked x10, 4-bit g64, s = 2 %, r = 4, T = 3, one attention output."""
    w = wl.WORKLOADS["tiny"]
    p, caches = _workload_encode_check(w, [(0, 0)], n_extra=0, nblk=1)
    op = oracle_params(p)
    xk, xv = wl.kv_unit_np(w, "k", 0, 0, 0), wl.kv_unit_np(w, "v", 0, 0, 0)
    assert np.abs(xk).max() > 10.0     # the spikes are there
    for c, x in ((caches["k"], xk), (caches["v"], xv)):
        o = oracle.encode_unit(x, op)
        compare_dense(c.dense().cpu().numpy()[0, 0], oracle.reconstruct_unit(o, op), o.scale, w.group, "tiny")
    q = wl.rows_torch(w, wl.S_Q, 0, 0, w.Hq, "cuda")
    tau = 1.0 / math.sqrt(128)
    out = gear.decode_attn(caches["k"], caches["v"], q, tau, out_dtype=torch.float32).cpu().numpy()
    ok, ov = oracle.Cache(op, 1, 1, 128), oracle.Cache(op, 1, 1, 128)
    ok.encode(xk[None, None])
    ov.encode(xv[None, None])
    ref = oracle.decode_attn(ok, ov, wl.rows_np(w, wl.S_Q, 0, 0, w.Hq), tau)
    assert np.abs(out - ref).max() <= 1e-3 * np.abs(ov.dense()).max()
    assert gear.device_status() == 0


def test_full_llama7b_layer_encode():
    w = wl.WORKLOADS["llama7b_layer_encode"]
    _workload_encode_check(w, _units_bh(w))


def test_full_llama7b_layer_encode_batch():
    """The K and V of the layer in one batched encode, as the benchmark runs it."""
    w = wl.WORKLOADS["llama7b_layer_encode"]
    p = _wparams(w)
    op = oracle_params(p)
    xs = [wl.kv_tensor_torch(w, which, 0, "cuda") for which in ["k", "v"]]
    cs = [gear.Cache(p, w.B, w.H, w.n, 1, TORCH_DT[w.dtype]) for _ in range(2)]
    gear.encode_batch(cs, xs)
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    _check_sampled_units(w, dict(zip(["k", "v"], cs)), _units_bh(w), op, p, 0, "batch")


def _decode_units_check(w, out, units, op, layer=0, tol=1e-3):
    """Attention of every query head of each sampled unit against the oracle's
    reconstruction of that unit (no buffer)."""
    qn = wl.rows_np(w, wl.S_Q, layer, 0, w.Hq)
    hq = w.Hq // w.H
    tau = 1.0 / math.sqrt(128)

    def ref(bh):
        b, h = bh
        K = oracle.reconstruct_unit(oracle.encode_unit(wl.kv_unit_np(w, "k", layer, b, h), op), op)
        V = oracle.reconstruct_unit(oracle.encode_unit(wl.kv_unit_np(w, "v", layer, b, h), op), op)
        return [oracle.attention(qn[b, j], K, V, tau) for j in range(h * hq, (h + 1) * hq)], np.abs(V).max()

    for (b, h), (refs, vmax) in zip(units, pmap(ref, units)):
        for j, r in zip(range(h * hq, (h + 1) * hq), refs):
            err = np.abs(out[b, j] - r).max()
            assert err <= tol * vmax, f"{w.name} layer {layer} unit ({b},{h}) head {j}: {err:.3e}"


def test_full_twobit_b64_encode_and_decode():
    w = wl.WORKLOADS["twobit_b64_ctx8192"]
    units = _units_bh(w)
    p, caches = _workload_encode_check(w, units)
    q = wl.rows_torch(w, wl.S_Q, 0, 0, w.Hq, "cuda")
    out = gear.decode_attn(caches["k"], caches["v"], q, 1.0 / math.sqrt(128), out_dtype=torch.float32).cpu().numpy()
    _decode_units_check(w, out, units, oracle_params(p))


def test_full_decode_b16_with_buffer_and_flush():
    w = wl.WORKLOADS["decode_b16_ctx8192"]
    p = _wparams(w)
    op = oracle_params(p)
    kc = gear.Cache(p, w.B, w.H, w.n + 64, 4, TORCH_DT[w.dtype])
    vc = gear.Cache(p, w.B, w.H, w.n + 64, 4, TORCH_DT[w.dtype])
    kc.encode(wl.kv_tensor_torch(w, "k", 0, "cuda"))
    vc.encode(wl.kv_tensor_torch(w, "v", 0, "cuda"))
    for i in range(w.buffer_fill):
        gear.append_buffer(kc, vc, wl.rows_torch(w, wl.S_KBUF, 0, i, w.H, "cuda"),
                           wl.rows_torch(w, wl.S_VBUF, 0, i, w.H, "cuda"))
    q = wl.rows_torch(w, wl.S_Q, 0, 0, w.Hq, "cuda")
    tau = 1.0 / math.sqrt(128)
    out = gear.decode_attn(kc, vc, q, tau, out_dtype=torch.float32).cpu().numpy()
    # one more token: flushes the full buffer as block 1
    gear.append_buffer(kc, vc, wl.rows_torch(w, wl.S_KNEW, 0, 0, w.H, "cuda"),
                       wl.rows_torch(w, wl.S_VNEW, 0, 0, w.H, "cuda"))
    out2 = gear.decode_attn(kc, vc, q, tau, out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    qn = wl.rows_np(w, wl.S_Q, 0, 0, w.Hq)
    units = _units_bh(w)
    _check_sampled_units(w, {"k": kc, "v": vc}, units, op, p, 0, "decode cache")

    def refs(bh):
        b, h = bh
        ok, ov = oracle.Cache(op, 1, 1, 128), oracle.Cache(op, 1, 1, 128)
        ok.encode(wl.kv_unit_np(w, "k", 0, b, h)[None, None])
        ov.encode(wl.kv_unit_np(w, "v", 0, b, h)[None, None])
        for i in range(w.buffer_fill):
            ok.append(wl.rows_np(w, wl.S_KBUF, 0, i, w.H)[b:b + 1, h:h + 1])
            ov.append(wl.rows_np(w, wl.S_VBUF, 0, i, w.H)[b:b + 1, h:h + 1])
        r1 = oracle.decode_attn(ok, ov, qn[b:b + 1, h:h + 1], tau)[0, 0]
        v1 = np.abs(ov.dense()).max()
        ok.append(wl.rows_np(w, wl.S_KNEW, 0, 0, w.H)[b:b + 1, h:h + 1])
        ov.append(wl.rows_np(w, wl.S_VNEW, 0, 0, w.H)[b:b + 1, h:h + 1])
        r2 = oracle.decode_attn(ok, ov, qn[b:b + 1, h:h + 1], tau)[0, 0]
        return r1, v1, r2, np.abs(ov.dense()).max(), ok.blocks[1][0]

    for (b, h), (r1, v1, r2, v2, blk1) in zip(units, pmap(refs, units)):
        assert np.abs(out[b, h] - r1).max() <= 1e-3 * v1, (b, h)
        assert np.abs(out2[b, h] - r2).max() <= 1e-3 * v2, (b, h)
        compare_unit(gpu_block(kc, b * w.H + h, w.n, w.n + w.buffer_len, 1, w.buffer_rank), blk1, p,
                     f"flushed K block ({b},{h})")


def test_full_llama3_gqa_all_layers():
    """The GQA cache of all 32 layers (8 kv heads shared by 32 query heads, bf16,
    32768 tokens, a full 20-token buffer): one decode step per layer, checked on one
    (b, h) unit per layer (a different one each layer) for every query head of its
    group, plus bit-exact codes of that unit."""
    w = wl.WORKLOADS["llama3_8b_gqa"]
    p = _wparams(w)
    op = oracle_params(p)
    tau = 1.0 / math.sqrt(128)
    hq = w.Hq // w.H
    kc = gear.Cache(p, w.B, w.H, w.n + 64, 4, TORCH_DT[w.dtype])
    vc = gear.Cache(p, w.B, w.H, w.n + 64, 4, TORCH_DT[w.dtype])
    outs, picks = [], []
    for layer in range(w.layers):
        for c in (kc, vc):
            c.reset()
        kc.encode(wl.kv_tensor_torch(w, "k", layer, "cuda"))
        vc.encode(wl.kv_tensor_torch(w, "v", layer, "cuda"))
        for i in range(w.buffer_fill):
            gear.append_buffer(kc, vc, wl.rows_torch(w, wl.S_KBUF, layer, i, w.H, "cuda"),
                               wl.rows_torch(w, wl.S_VBUF, layer, i, w.H, "cuda"))
        q = wl.rows_torch(w, wl.S_Q, layer, 0, w.Hq, "cuda")
        out = gear.decode_attn(kc, vc, q, tau, out_dtype=torch.float32).cpu().numpy()
        b, h = layer % w.B, (3 * layer + 1) % w.H
        u = b * w.H + h
        picks.append((layer, b, h))
        outs.append((out[b, h * hq:(h + 1) * hq], gpu_block(kc, u, 0, w.n, 0, w.rank)))
    torch.cuda.synchronize()
    assert gear.device_status() == 0

    def ref(lbh):
        layer, b, h = lbh
        ok, ov = oracle.Cache(op, 1, 1, 128), oracle.Cache(op, 1, 1, 128)
        ok.encode(wl.kv_unit_np(w, "k", layer, b, h)[None, None])
        ov.encode(wl.kv_unit_np(w, "v", layer, b, h)[None, None])
        for i in range(w.buffer_fill):
            ok.append(wl.rows_np(w, wl.S_KBUF, layer, i, w.H)[b:b + 1, h:h + 1])
            ov.append(wl.rows_np(w, wl.S_VBUF, layer, i, w.H)[b:b + 1, h:h + 1])
        qn = wl.rows_np(w, wl.S_Q, layer, 0, w.Hq)[b:b + 1, h * hq:(h + 1) * hq]
        return oracle.decode_attn(ok, ov, qn, tau)[0], np.abs(ov.dense()).max(), ok.blocks[0][0]

    for (layer, b, h), (got, gk), (r, vmax, kunit) in zip(picks, outs, pmap(ref, picks)):
        err = np.abs(got - r).max()
        assert err <= 8e-3 * vmax, f"layer {layer} unit ({b},{h}): {err:.3e} > {8e-3 * vmax:.3e}"
        compare_unit(gk, kunit, p, f"layer {layer} K ({b},{h})")
