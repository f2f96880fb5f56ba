"""GPU parity of the KIVI-combined key quantizer (per-channel groups of g tokens,
outliers per token, low rank of the residual) against the CPU oracle: codes,
per-channel scales and zero points and outliers bit for bit, the low-rank term
and the reconstruction within the tolerances of the per-token codec."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TORCH_DT, compare_dense, oracle_params, seeded_kv, to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_compression_gear_b200 as gear
else:
    gear = None


def ch_block(cache, u, t0, t1, slot0, rank, blk=0):
    """Stored arrays of tokens [t0, t1) of unit u (block blk), whose token groups start at slot0."""
    A = cache.arrays()
    g = cache.c.p.group_size
    n = t1 - t0
    ng = (n + g - 1) // g
    e = 0
    while (2 << e) <= n:
        e += 1
    e //= 2
    m = A["meta"][u, slot0:slot0 + ng].cpu().numpy()
    return {
        "codes": A["codes"][u, t0:t1].cpu().numpy(),
        "scale": m[..., 0], "zero": m[..., 1],
        "oidx": A["oidx"][u, t0:t1].cpu().numpy(),
        "oval": A["oval"][u, t0:t1].float().cpu().numpy(),
        "L": A["lfac"][u, t0:t1, :rank].float().cpu().numpy().astype(np.float64) * 2.0 ** -e,
        "Rf": A["rfac"][u, blk, :, :rank].cpu().numpy().astype(np.float64) * 2.0 ** e,
    }


def compare_ch(gb, o, blk, what):
    k = o.oidx.shape[1]
    assert np.array_equal(gb["codes"].view(np.uint32), o.codes), f"{what}: codes differ"
    assert np.array_equal(gb["scale"].view(np.uint32), o.scale.view(np.uint32)), f"{what}: scale differs"
    assert np.array_equal(gb["zero"].view(np.uint32), o.zero.view(np.uint32)), f"{what}: zero differs"
    if k:
        assert np.array_equal(gb["oidx"][:, :k].astype(np.int32), o.oidx), f"{what}: outlier index"
        assert np.array_equal(gb["oval"][:, :k].view(np.uint32), o.oval.view(np.uint32)), f"{what}: outlier value"
    if o.rank:
        lr = gb["L"] @ gb["Rf"].T
        err = np.abs(lr - o.L @ o.Rf.T).max()
        rmax = np.abs(o.resid).max()
        assert err <= 1e-3 * rmax + 1e-30, f"{what}: L Rf^T error {err:.3e} > {1e-3 * rmax:.3e}"


KIVI_ENC_CASES = [
    # dtype, B, H, n, bits, g, s, r
    ("f16", 1, 2, 300, 4, 64, 0.02, 4),    # the last group has 44 tokens
    ("bf16", 2, 1, 256, 2, 32, 0.05, 8),
    ("f16", 1, 2, 128, 8, 128, 0.02, 4),
    ("f16", 1, 1, 20, 4, 32, 0.02, 2),     # one short group
    ("bf16", 1, 3, 513, 4, 32, 0.0, 4),    # GEAR-L with per-channel keys
]


@pytest.mark.parametrize("dtype,B,H,n,bits,g,s,r", KIVI_ENC_CASES)
def test_kivi_encode_matches_oracle(dtype, B, H, n, bits, g, s, r):
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, power_iters=3, buffer_len=2 * g,
                         buffer_rank=2, seed=71 + n, channel_groups=True)
    x = seeded_kv(19 + n, 1, (B, H, n, 128), dtype, channel_scale=True)
    kc = gear.Cache(p, B, H, n + 32, 2, TORCH_DT[dtype])
    kc.encode(to_dev(x, dtype))
    dense = kc.dense().cpu().numpy()
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    op = oracle_params(p)
    for u in range(B * H):
        o = oracle.encode_unit(x[u // H, u % H], op)
        compare_ch(ch_block(kc, u, 0, n, 0, r), o, 0, f"unit {u}")
        grp = np.arange(n) // g
        compare_dense(dense[u // H, u % H], oracle.reconstruct_unit(o, op), o.scale[grp], 1, f"unit {u}")


def test_kivi_flush_blocks_match_oracle():
    """Appends flush whole groups (n_b = 2g) into blocks that follow a block 0 ending in
    a short group; every flushed key block equals the oracle's."""
    dtype, B, H, n0, g = "f16", 1, 2, 100, 32
    p = gear.make_params(bits=4, group_size=g, outlier_frac=0.05, rank=4, power_iters=3, buffer_len=2 * g,
                         buffer_rank=2, seed=3, channel_groups=True)
    pv = gear.make_params(bits=4, group_size=g, outlier_frac=0.05, rank=4, power_iters=3, buffer_len=2 * g,
                          buffer_rank=2, seed=3)
    nap = 4 * g + 5
    xk = seeded_kv(5, 1, (B, H, n0, 128), dtype, channel_scale=True)
    xv = seeded_kv(5, 2, (B, H, n0, 128), dtype)
    kc = gear.Cache(p, B, H, n0 + nap + 1, 4, TORCH_DT[dtype])
    vc = gear.Cache(pv, B, H, n0 + nap + 1, 4, TORCH_DT[dtype])
    kc.encode(to_dev(xk, dtype))
    vc.encode(to_dev(xv, dtype))
    ok = oracle.Cache(oracle_params(p), B, H, 128)
    ok.encode(xk)
    for i in range(nap):
        rk = seeded_kv(200 + i, 3, (B, H, 128), dtype)
        rv = seeded_kv(200 + i, 4, (B, H, 128), dtype)
        gear.append_buffer(kc, vc, to_dev(rk, dtype), to_dev(rv, dtype))
        ok.append(rk)
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    assert kc.n_comp == ok.n_comp and kc.n_blk == len(ok.blocks) == 3
    slot = -(-n0 // g)
    t0 = n0
    for bi in (1, 2):
        for u in range(B * H):
            compare_ch(ch_block(kc, u, t0, t0 + 2 * g, slot, 2, bi), ok.blocks[bi][u], bi, f"block {bi} unit {u}")
        t0 += 2 * g
        slot += 2


KIVI_DEC_CASES = [
    # dtype, B, H, Hq, n0, nappend, bits, g, s, r
    ("f16", 2, 2, 4, 300, 70, 4, 32, 0.02, 4),    # flushes of 64 tokens after a short last group
    ("bf16", 1, 2, 2, 257, 3, 2, 64, 0.05, 8),
    ("f16", 2, 1, 1, 130, 129, 4, 64, 0.0, 4),    # GEAR-L keys, one flush of 128 tokens
    ("bf16", 1, 2, 8, 64, 40, 4, 32, 0.02, 4),    # four query heads per kv head
]


@pytest.mark.parametrize("dtype,B,H,Hq,n0,nappend,bits,g,s,r", KIVI_DEC_CASES)
def test_kivi_decode_matches_oracle(dtype, B, H, Hq, n0, nappend, bits, g, s, r):
    """Decode attention over a K cache with per-channel key groups and a V cache with
    per-token groups (the KIVI combination: keys per channel, values per token)."""
    common = dict(bits=bits, group_size=g, outlier_frac=s, rank=r, power_iters=3, buffer_len=2 * g,
                  buffer_rank=2, seed=13)
    pk = gear.make_params(channel_groups=True, **common)
    pv = gear.make_params(**common)
    xk = seeded_kv(31 + n0, 1, (B, H, n0, 128), dtype, channel_scale=True)
    xv = seeded_kv(31 + n0, 2, (B, H, n0, 128), dtype)
    n_max, nblk = n0 + nappend + 1, 2 + nappend // (2 * g)
    kc = gear.Cache(pk, B, H, n_max, nblk, TORCH_DT[dtype])
    vc = gear.Cache(pv, B, H, n_max, nblk, TORCH_DT[dtype])
    kc.encode(to_dev(xk, dtype))
    vc.encode(to_dev(xv, dtype))
    ok, ov = oracle.Cache(oracle_params(pk), B, H, 128), oracle.Cache(oracle_params(pv), B, H, 128)
    ok.encode(xk)
    ov.encode(xv)
    for i in range(nappend):
        rk = seeded_kv(400 + i, 3, (B, H, 128), dtype)
        rv = seeded_kv(400 + i, 4, (B, H, 128), dtype)
        gear.append_buffer(kc, vc, to_dev(rk, dtype), to_dev(rv, dtype))
        ok.append(rk)
        ov.append(rv)
    torch.cuda.synchronize()
    assert kc.n_comp == ok.n_comp and kc.n_blk == len(ok.blocks)
    q = seeded_kv(90 + n0, 5, (B, Hq, 128), dtype)
    tau = 1.0 / math.sqrt(128)
    ref = oracle.decode_attn(ok, ov, q, tau)
    vmax = np.abs(ov.dense()).max()
    tol = 8e-3 if dtype == "bf16" else 1e-3
    for out_dt in (TORCH_DT[dtype], torch.float32):
        out = gear.decode_attn(kc, vc, to_dev(q, dtype), tau, out_dtype=out_dt).float().cpu().numpy()
        err = np.abs(out - ref).max()
        assert err <= tol * vmax, f"attention error {err:.3e} > {tol * vmax:.3e}"
    assert gear.device_status() == 0
