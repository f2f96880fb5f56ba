"""GPU parity of the paged layout: rows (sequences) with their own prompt
lengths join, append and leave independently, each row's buffer flushing when
that row's buffer is full. The oracle of a batch of independent rows is one
oracle cache per row (batch 1), driven by the same calls; the stored blocks are
compared bit for bit (codes, scales, zero points, outliers) and attention within
the decode tolerance. With equal rows the paged cache must store exactly what
the contiguous cache stores."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as wl
from tests.gpu_helpers import TORCH_DT, compare_unit, oracle_params, pmap, seeded_kv, spread_units, to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_compression_gear_b200 as gear
else:
    gear = None

TAU = 1.0 / math.sqrt(128)


def _tol_out(dtype: str) -> float:
    return 8e-3 if dtype == "bf16" else 1e-3


def paged_block(cache, b: int, h: int, t0: int, t1: int, blk: int, rank: int) -> dict:
    """Stored arrays of tokens [t0, t1) of row b, head h, gathered through the
    host copy of the block table (numpy; L and Rf unscaled)."""
    A = cache.arrays()
    P = cache.c.page_tokens
    _, _, _, table = cache.counters()
    t = np.arange(t0, t1)
    pg = table[b, t // P]
    assert (pg >= 0).all()
    off = t % P
    n = t1 - t0
    e = 0
    while (2 << e) <= n:
        e += 1
    e //= 2
    # host-side bounds first: a bad index fails here, not in a device-side check
    assert pg.max() < A["codes"].shape[0] and h < A["codes"].shape[1] and off.max() < A["codes"].shape[2]
    assert blk < A["rfac"].shape[2] and b < A["rfac"].shape[0]
    pg_t = torch.from_numpy(pg.astype(np.int64)).cuda()
    off_t = torch.from_numpy(off.astype(np.int64)).cuda()

    def take(name):
        return A[name][pg_t, h, off_t].cpu()

    if cache.c.p.channel_groups:
        meta = None   # per-unit token-group slots, not per-token rows: see paged_ch_block
    else:
        meta = take("meta").float().numpy() if A["meta"].dtype == torch.float16 else take("meta").numpy()
    return {
        "codes": take("codes").numpy(),
        "meta": meta,
        "oidx": take("oidx").numpy(),
        "oval": take("oval").float().numpy(),
        "L": take("lfac")[:, :rank].float().numpy().astype(np.float64) * 2.0 ** -e,
        "Rf": A["rfac"][b, h, blk, :, :rank].cpu().numpy().astype(np.float64) * 2.0 ** e,
    }


class RowOracle:
    """One oracle K and V cache (batch 1) per row of the paged batch (opv: the
    V parameters when they differ from K's)."""

    def __init__(self, op, B, H, opv=None):
        self.op, self.opv, self.H = op, opv or op, H
        self.k = [None] * B
        self.v = [None] * B

    def encode(self, b, xk, xv):
        self.k[b] = oracle.Cache(self.op, 1, self.H, 128)
        self.v[b] = oracle.Cache(self.opv, 1, self.H, 128)
        self.k[b].encode(xk[None])
        self.v[b].encode(xv[None])

    def append(self, b, rk, rv):
        self.k[b].append(rk[None])
        self.v[b].append(rv[None])

    def release(self, b):
        self.k[b] = self.v[b] = None

    def attn(self, q):
        out = np.zeros(q.shape, dtype=np.float64)
        vmax = 0.0
        for b in range(q.shape[0]):
            if self.k[b] is None:
                continue
            out[b] = oracle.decode_attn(self.k[b], self.v[b], q[b:b + 1], TAU)[0]
            vmax = max(vmax, float(np.abs(self.v[b].dense()).max()))
        return out, vmax


def _check_blocks(kc, ro: RowOracle, B, H, p, what):
    b0, nblk, nbuf, _ = kc.counters()
    for b in range(B):
        if ro.k[b] is None:
            assert nblk[b] == 0 and nbuf[b] == 0
            continue
        ok = ro.k[b]
        assert nblk[b] == len(ok.blocks) and nbuf[b] == len(ok.buffer), (what, b)
        t0 = 0
        for bi, blk in enumerate(ok.blocks):
            n = blk[0].codes.shape[0]
            rank = p.rank if bi == 0 else p.buffer_rank
            for h in range(H):
                compare_unit(paged_block(kc, b, h, t0, t0 + n, bi, rank), blk[h], p, f"{what} row {b} block {bi}")
            t0 += n
        assert b0[b] == ok.blocks[0][0].codes.shape[0]


PAGED_CASES = [
    # dtype, H, Hq, bits, g, s, r, n_b, r_buf, P, meta_f16
    ("f16", 2, 4, 4, 64, 0.02, 4, 24, 2, 64, False),
    ("bf16", 2, 16, 2, 32, 0.05, 8, 20, 2, 32, False),   # eight query heads per kv head, pages of one tile
    ("f32", 1, 2, 8, 64, 0.02, 2, 12, 1, 96, False),
    ("f16", 2, 2, 4, 32, 0.0, 4, 16, 2, 64, True),       # GEAR-L, binary16 metadata
]


@pytest.mark.parametrize("dtype,H,Hq,bits,g,s,r,n_b,r_buf,P,meta_f16", PAGED_CASES)
def test_paged_rows_match_oracle(dtype, H, Hq, bits, g, s, r, n_b, r_buf, P, meta_f16):
    B = 4
    p = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=r, buffer_len=n_b, buffer_rank=r_buf,
                         power_iters=3, seed=23, meta_f16=meta_f16)
    op = oracle_params(p)
    ppr, num_pages = 8, 20
    kc = gear.PagedCache(p, B, H, P, num_pages, ppr, 8, TORCH_DT[dtype])
    vc = gear.PagedCache(p, B, H, P, num_pages, ppr, 8, TORCH_DT[dtype])
    ro = RowOracle(op, B, H)
    seed = [1000]

    def kv(n, rows):
        seed[0] += 1
        xk = seeded_kv(seed[0], 1, (rows, H, n, 128), dtype, channel_scale=True)
        xv = seeded_kv(seed[0], 2, (rows, H, n, 128), dtype)
        return xk, xv

    def encode(rows, n):
        xk, xv = kv(n, len(rows))
        kc.encode_rows(rows, to_dev(xk, dtype))
        vc.encode_rows(rows, to_dev(xv, dtype))
        for i, b in enumerate(rows):
            ro.encode(b, xk[i], xv[i])

    def append(rows):
        seed[0] += 1
        rk = seeded_kv(seed[0], 3, (len(rows), H, 128), dtype)
        rv = seeded_kv(seed[0], 4, (len(rows), H, 128), dtype)
        gear.append_rows(kc, vc, rows, to_dev(rk, dtype), to_dev(rv, dtype))
        for i, b in enumerate(rows):
            ro.append(b, rk[i], rv[i])

    def check(what):
        torch.cuda.synchronize()
        assert gear.device_status() == 0
        seed[0] += 1
        q = seeded_kv(seed[0], 5, (B, Hq, 128), dtype)
        od, vmax = ro.attn(q)
        out = gear.decode_attn(kc, vc, to_dev(q, dtype), TAU, out_dtype=torch.float32).cpu().numpy()
        err = np.abs(out - od).max()
        assert err <= _tol_out(dtype) * vmax, f"{what}: attention error {err:.3e} vs {_tol_out(dtype) * vmax:.3e}"
        for b in range(B):
            if ro.k[b] is None:
                assert not out[b].any(), f"{what}: row {b} has no tokens"
        _check_blocks(kc, ro, B, H, p, what)
        assert np.array_equal(kc.host, vc.host)

    # rows 0 and 2 join with 100 tokens, row 1 with 37; row 3 stays empty
    encode([0, 2], 100)
    encode([1], 37)
    check("after prefill")
    for step in range(60):
        rows = [0] + ([1] if step % 2 == 0 else []) + ([2] if step % 3 == 0 else []) + ([3] if step >= 21 else [])
        if step == 20:
            encode([3], 70)
        if step == 40:   # row 1 leaves; its pages go back to the pool and a new sequence takes the row
            kc.release_rows([1])
            vc.release_rows([1])
            ro.release(1)
            check("after release")
            encode([1], 50)
        append(rows)
        if step in (25, 49, 59):
            check(f"step {step}")
    b0, nblk, nbuf, _ = kc.counters()
    assert nblk.max() >= 3   # some row flushed twice
    assert len(set(nblk.tolist())) > 1   # rows at different block counts
    # every page is accounted for
    _, _, _, table = kc.counters()
    used = table[table >= 0]
    assert len(set(used.tolist())) == used.size
    assert used.size + kc.free_pages() == num_pages


@pytest.mark.parametrize("dtype,Hq", [("f16", 4), ("bf16", 2)])
def test_paged_equal_rows_match_contiguous_exactly(dtype, Hq):
    """Equal rows: the paged cache runs the same encoder launches (same unit
    count and tiling) and the same decode plan, so every stored value is
    bit-identical to the contiguous cache's, and attention agrees up to the
    order of the value-outlier atomics (fp32 sums in either order)."""
    B, H, n0, n_b = 3, 2, 150, 20
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, buffer_len=n_b, buffer_rank=2,
                         power_iters=3, seed=5)
    xk = seeded_kv(71, 1, (B, H, n0, 128), dtype, channel_scale=True)
    xv = seeded_kv(71, 2, (B, H, n0, 128), dtype)
    kc = gear.Cache(p, B, H, 256, 6, TORCH_DT[dtype])
    vc = gear.Cache(p, B, H, 256, 6, TORCH_DT[dtype])
    pk = gear.PagedCache(p, B, H, 64, 16, 4, 6, TORCH_DT[dtype])
    pv = gear.PagedCache(p, B, H, 64, 16, 4, 6, TORCH_DT[dtype])
    kc.encode(to_dev(xk, dtype))
    vc.encode(to_dev(xv, dtype))
    pk.encode_rows([0, 1, 2], to_dev(xk, dtype))
    pv.encode_rows([0, 1, 2], to_dev(xv, dtype))
    for i in range(45):
        rk = to_dev(seeded_kv(300 + i, 3, (B, H, 128), dtype), dtype)
        rv = to_dev(seeded_kv(300 + i, 4, (B, H, 128), dtype), dtype)
        gear.append_buffer(kc, vc, rk, rv)
        gear.append_rows(pk, pv, [0, 1, 2], rk, rv)
        if i in (0, 20, 44):
            q = to_dev(seeded_kv(900 + i, 5, (B, Hq, 128), dtype), dtype)
            a = gear.decode_attn(kc, vc, q, TAU, out_dtype=torch.float32)
            b = gear.decode_attn(pk, pv, q, TAU, out_dtype=torch.float32)
            assert (a - b).abs().max().item() <= 1e-5 * a.abs().max().item() + 1e-30, i
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    assert (pk.n_comp, pk.n_buf, pk.c.n_blk) == (kc.n_comp, kc.n_buf, kc.n_blk)
    A, Pa = kc.arrays(), pk.arrays()
    _, _, _, table = pk.counters()
    P = pk.c.page_tokens
    t = np.arange(kc.n_comp)
    for b in range(B):
        pg = torch.from_numpy(table[b, t // P].astype(np.int64)).cuda()
        off = torch.from_numpy((t % P).astype(np.int64)).cuda()
        for h in range(H):
            u = b * H + h
            for name in ("codes", "meta", "oidx", "oval", "lfac"):
                assert torch.equal(A[name][u, :kc.n_comp], Pa[name][pg, h, off]), (name, b, h)
            assert torch.equal(A["rfac"][u, :kc.n_blk], Pa["rfac"][b, h, :kc.n_blk]), (b, h)
            assert torch.equal(A["buf"][u], Pa["buf"][b, h])


def test_paged_pool_exhaustion_and_reuse():
    B, H = 3, 1
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=2, buffer_len=8, buffer_rank=1)
    kc = gear.PagedCache(p, B, H, 32, 5, 4, 8, torch.float16)
    vc = gear.PagedCache(p, B, H, 32, 5, 4, 8, torch.float16)
    x = to_dev(seeded_kv(3, 1, (1, H, 64, 128), "f16"), "f16")
    kc.encode_rows([0], x)      # 2 pages
    vc.encode_rows([0], x)
    kc.encode_rows([1], x)      # 2 pages
    vc.encode_rows([1], x)
    assert kc.free_pages() == 1
    with pytest.raises(gear.GearError) as ei:
        kc.encode_rows([2], x)  # needs 2, 1 left
    assert ei.value.status == gear.gear.GEAR_ERR_CAPACITY
    with pytest.raises(gear.GearError) as ei:
        kc.encode_rows([0], x)  # row 0 is not empty
    assert ei.value.status == gear.gear.GEAR_ERR_INVALID_ARG
    with pytest.raises(gear.GearError) as ei:
        gear.append_rows(kc, vc, [2], x[0, :, 0].contiguous(), x[0, :, 0].contiguous())   # row 2 never encoded
    assert ei.value.status == gear.gear.GEAR_ERR_INVALID_ARG
    # fill row 0's buffer (8 tokens), then the ninth append flushes into the last free page
    r = x[0, :, :1].reshape(1, H, 128).contiguous()
    for _ in range(9):
        gear.append_rows(kc, vc, [0], r, r)
    assert kc.free_pages() == 0
    # row 1's flush would need a page: nothing is enqueued and the counters stay
    for _ in range(8):
        gear.append_rows(kc, vc, [1], r, r)
    before = kc.host.copy()
    with pytest.raises(gear.GearError) as ei:
        gear.append_rows(kc, vc, [1], r, r)
    assert ei.value.status == gear.gear.GEAR_ERR_CAPACITY
    assert np.array_equal(kc.host, before)
    kc.release_rows([0])
    vc.release_rows([0])
    assert kc.free_pages() == 3
    gear.append_rows(kc, vc, [1], r, r)   # the flush takes a page row 0 gave back
    kc.encode_rows([2], x)
    vc.encode_rows([2], x)
    assert kc.free_pages() == 0
    q = to_dev(seeded_kv(4, 5, (B, H, 128), "f16"), "f16")
    out = gear.decode_attn(kc, vc, q, TAU, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    assert not out[0].any() and out[1].abs().max() > 0 and out[2].abs().max() > 0


def test_paged_many_ragged_rows_match_oracle():
    """More rows than a warp has lanes (the decoder's row search runs in passes of
    32 rows), lengths from 1 to a few hundred tokens, empty rows between them, and
    buffers at different fills: every row against its own oracle caches."""
    B, H, Hq, dtype = 45, 1, 2, "f16"
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=1, buffer_len=8, buffer_rank=1,
                         power_iters=2, seed=9)
    op = oracle_params(p)
    kc = gear.PagedCache(p, B, H, 32, 400, 12, 6, torch.float16)
    vc = gear.PagedCache(p, B, H, 32, 400, 12, 6, torch.float16)
    ro = RowOracle(op, B, H)
    lengths = [0 if b % 7 == 3 else 1 + (b * 37) % 300 for b in range(B)]
    for b, n in enumerate(lengths):
        if n == 0:
            continue
        xk = seeded_kv(500 + b, 1, (1, H, n, 128), dtype, channel_scale=True)
        xv = seeded_kv(500 + b, 2, (1, H, n, 128), dtype)
        kc.encode_rows([b], to_dev(xk, dtype))
        vc.encode_rows([b], to_dev(xv, dtype))
        ro.encode(b, xk[0], xv[0])
    live = [b for b in range(B) if lengths[b]]
    for step in range(20):
        rows = [b for b in live if (b + step) % 3 != 0]
        rk = seeded_kv(700 + step, 3, (len(rows), H, 128), dtype)
        rv = seeded_kv(700 + step, 4, (len(rows), H, 128), dtype)
        gear.append_rows(kc, vc, rows, to_dev(rk, dtype), to_dev(rv, dtype))
        for i, b in enumerate(rows):
            ro.append(b, rk[i], rv[i])
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    q = seeded_kv(901, 5, (B, Hq, 128), dtype)
    od, vmax = ro.attn(q)
    for _ in range(2):   # twice: nothing depends on what the workspace held before
        out = gear.decode_attn(kc, vc, to_dev(q, dtype), TAU, out_dtype=torch.float32).cpu().numpy()
        err = np.abs(out - od).max()
        assert err <= 1e-3 * vmax, f"attention error {err:.3e} vs {1e-3 * vmax:.3e}"
    for b in range(B):
        if not lengths[b]:
            assert not out[b].any()
    _check_blocks(kc, ro, B, H, p, "many rows")


def test_paged_pair_must_agree():
    """K and V caches whose pages were handed out in different orders are
    refused by decode and append (one table serves both tensors)."""
    B, H = 2, 1
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=2, buffer_len=8, buffer_rank=1)
    kc = gear.PagedCache(p, B, H, 32, 8, 4, 4, torch.float16)
    vc = gear.PagedCache(p, B, H, 32, 8, 4, 4, torch.float16)
    x = to_dev(seeded_kv(8, 1, (1, H, 40, 128), "f16"), "f16")
    kc.encode_rows([0], x)
    kc.encode_rows([1], x)
    vc.encode_rows([1], x)   # the other order: same counters, other pages
    vc.encode_rows([0], x)
    b0k, nbk, nfk, tk = kc.counters()
    b0v, nbv, nfv, tv = vc.counters()
    assert (b0k == b0v).all() and (nbk == nbv).all() and (nfk == nfv).all() and not (tk == tv).all()
    q = to_dev(seeded_kv(9, 5, (B, H, 128), "f16"), "f16")
    with pytest.raises(gear.GearError) as ei:
        gear.decode_attn(kc, vc, q, TAU)
    assert ei.value.status == gear.gear.GEAR_ERR_INVALID_ARG
    r = x[0, :, :1].reshape(1, H, 128).contiguous()
    with pytest.raises(gear.GearError) as ei:
        gear.append_rows(kc, vc, [0], r, r)
    assert ei.value.status == gear.gear.GEAR_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert gear.device_status() == 0


def test_full_paged_decode_b16_ragged():
    """The batch-16 decode workload in the launch configuration the benchmark's
    paged line times (pages of 256 tokens): rows' prompts spread over 4096..8192
    tokens, a full 20-token buffer, decode; then one more token per row, which
    flushes every row's buffer as its block 1 (mid-page), and decode again. 16
    sampled (row, head) units against the oracle built from the same tokens."""
    w = wl.WORKLOADS["decode_b16_ctx8192"]
    p = gear.make_params(bits=w.bits, group_size=w.group, outlier_frac=w.s, rank=w.rank, power_iters=w.iters,
                         buffer_len=w.buffer_len, buffer_rank=w.buffer_rank, seed=w.seed)
    op = oracle_params(p)
    dt = TORCH_DT[w.dtype]
    P = 256
    ppr = -(-(w.n + 2 * w.buffer_len) // P)
    kc = gear.PagedCache(p, w.B, w.H, P, w.B * ppr, ppr, 4, dt)
    vc = gear.PagedCache(p, w.B, w.H, P, w.B * ppr, ppr, 4, dt)
    lengths = [w.n // 2 + (w.n // 2) * b // (w.B - 1) // 32 * 32 for b in range(w.B)]
    xs = {which: wl.kv_tensor_torch(w, which, 0, "cuda") for which in ("k", "v")}
    by_len = {}
    for b, n in enumerate(lengths):
        by_len.setdefault(n, []).append(b)
    for n, rs in by_len.items():
        kc.encode_rows(rs, xs["k"][rs][:, :, :n].contiguous())
        vc.encode_rows(rs, xs["v"][rs][:, :, :n].contiguous())
    del xs
    rows = list(range(w.B))
    for i in range(w.buffer_fill):
        gear.append_rows(kc, vc, rows, wl.rows_torch(w, wl.S_KBUF, 0, i, w.H, "cuda"),
                         wl.rows_torch(w, wl.S_VBUF, 0, i, w.H, "cuda"))
    q = wl.rows_torch(w, wl.S_Q, 0, 0, w.Hq, "cuda")
    out = gear.decode_attn(kc, vc, q, TAU, out_dtype=torch.float32).cpu().numpy()
    gear.append_rows(kc, vc, rows, wl.rows_torch(w, wl.S_KNEW, 0, 0, w.H, "cuda"),
                     wl.rows_torch(w, wl.S_VNEW, 0, 0, w.H, "cuda"))
    out2 = gear.decode_attn(kc, vc, q, TAU, out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    _, nblk, nbuf, _ = kc.counters()
    assert (nblk == 2).all() and (nbuf == 1).all()
    qn = wl.rows_np(w, wl.S_Q, 0, 0, w.Hq)
    units = [(u // w.H, u % w.H) for u in spread_units(w.B * w.H, 16)]

    def refs(bh):
        b, h = bh
        n = lengths[b]
        ok, ov = oracle.Cache(op, 1, 1, 128), oracle.Cache(op, 1, 1, 128)
        ok.encode(wl.kv_unit_np(w, "k", 0, b, h)[:n][None, None])
        ov.encode(wl.kv_unit_np(w, "v", 0, b, h)[:n][None, None])
        for i in range(w.buffer_fill):
            ok.append(wl.rows_np(w, wl.S_KBUF, 0, i, w.H)[b:b + 1, h:h + 1])
            ov.append(wl.rows_np(w, wl.S_VBUF, 0, i, w.H)[b:b + 1, h:h + 1])
        r1 = oracle.decode_attn(ok, ov, qn[b:b + 1, h:h + 1], TAU)[0, 0]
        v1 = np.abs(ov.dense()).max()
        ok.append(wl.rows_np(w, wl.S_KNEW, 0, 0, w.H)[b:b + 1, h:h + 1])
        ov.append(wl.rows_np(w, wl.S_VNEW, 0, 0, w.H)[b:b + 1, h:h + 1])
        r2 = oracle.decode_attn(ok, ov, qn[b:b + 1, h:h + 1], TAU)[0, 0]
        return r1, v1, r2, np.abs(ov.dense()).max(), ok.blocks[0][0], ok.blocks[1][0]

    for (b, h), (r1, v1, r2, v2, blk0, blk1) in zip(units, pmap(refs, units)):
        n = lengths[b]
        assert np.abs(out[b, h] - r1).max() <= 1e-3 * v1, (b, h)
        assert np.abs(out2[b, h] - r2).max() <= 1e-3 * v2, (b, h)
        compare_unit(paged_block(kc, b, h, 0, n, 0, w.rank), blk0, p, f"paged K block 0 ({b},{h})")
        compare_unit(paged_block(kc, b, h, n, n + w.buffer_len, 1, w.buffer_rank), blk1, p,
                     f"paged K block 1 ({b},{h})")


def paged_ch_block(cache, b, h, t0, t1, blk, rank, slot0):
    """Like paged_block, for a K cache with per-channel key groups: the block's
    token-group slots from slot0 (per unit) instead of per-token meta rows."""
    g = paged_block(cache, b, h, t0, t1, blk, rank)
    gs = cache.c.p.group_size
    ng = (t1 - t0 + gs - 1) // gs
    m = cache.arrays()["meta"][b, h, slot0:slot0 + ng].cpu().numpy()
    g["scale"], g["zero"] = m[..., 0], m[..., 1]
    return g


@pytest.mark.parametrize("dtype,bits,g,s", [("f16", 4, 32, 0.02), ("bf16", 2, 64, 0.05)])
def test_paged_kivi_keys_match_oracle(dtype, bits, g, s):
    """Per-channel key groups (the KIVI-combined quantizer) on the paged K cache,
    per-token groups on V: ragged prompts (block 0 ending in a short group),
    ragged appends and flushes of whole groups at different steps per row."""
    from tests.test_gpu_kivi import compare_ch
    B, H, Hq, n_b, P = 3, 2, 4, 2 * g, 64
    pk = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=4, buffer_len=n_b, buffer_rank=2,
                          power_iters=3, seed=31, channel_groups=True)
    pv = gear.make_params(bits=bits, group_size=g, outlier_frac=s, rank=4, buffer_len=n_b, buffer_rank=2,
                          power_iters=3, seed=31)
    kc = gear.PagedCache(pk, B, H, P, 40, 8, 6, TORCH_DT[dtype])
    vc = gear.PagedCache(pv, B, H, P, 40, 8, 6, TORCH_DT[dtype])
    ro = RowOracle(oracle_params(pk), B, H, oracle_params(pv))
    for rows, n in (([0, 1], 100), ([2], 45)):
        xk = seeded_kv(40 + n, 1, (len(rows), H, n, 128), dtype, channel_scale=True)
        xv = seeded_kv(40 + n, 2, (len(rows), H, n, 128), dtype)
        kc.encode_rows(rows, to_dev(xk, dtype))
        vc.encode_rows(rows, to_dev(xv, dtype))
        for i, b in enumerate(rows):
            ro.encode(b, xk[i], xv[i])
    for step in range(2 * n_b + 10):
        rows = [0] + ([1] if step % 2 == 0 else []) + ([2] if step >= 5 else [])
        rk = seeded_kv(600 + step, 3, (len(rows), H, 128), dtype)
        rv = seeded_kv(600 + step, 4, (len(rows), H, 128), dtype)
        gear.append_rows(kc, vc, rows, to_dev(rk, dtype), to_dev(rv, dtype))
        for i, b in enumerate(rows):
            ro.append(b, rk[i], rv[i])
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    _, nblk, nbuf, _ = kc.counters()
    assert nblk[0] >= 3 and len(set(nblk.tolist())) > 1
    for b in range(B):
        ok, ov = ro.k[b], ro.v[b]
        assert nblk[b] == len(ok.blocks) and nbuf[b] == len(ok.buffer)
        t0, slot = 0, 0
        for bi, (kb, vb) in enumerate(zip(ok.blocks, ov.blocks)):
            n = kb[0].codes.shape[0]
            rank = 4 if bi == 0 else 2
            for h in range(H):
                compare_ch(paged_ch_block(kc, b, h, t0, t0 + n, bi, rank, slot), kb[h], bi,
                           f"K row {b} block {bi} head {h}")
                compare_unit(paged_block(vc, b, h, t0, t0 + n, bi, rank), vb[h], pv, f"V row {b} block {bi}")
            t0 += n
            slot += (n + g - 1) // g
    q = seeded_kv(77, 5, (B, Hq, 128), dtype)
    od, vmax = ro.attn(q)
    out = gear.decode_attn(kc, vc, to_dev(q, dtype), TAU, out_dtype=torch.float32).cpu().numpy()
    err = np.abs(out - od).max()
    assert err <= _tol_out(dtype) * vmax, f"attention error {err:.3e} vs {_tol_out(dtype) * vmax:.3e}"


def _poison(cache, names=("codes", "meta", "oidx", "oval", "lfac", "rfac", "buf")):
    """Every byte of the cache's data arrays set to 0xFF (NaN for floats), so that
    a read of anything the library did not write shows in the result."""
    A = cache.arrays()
    for n in names:
        A[n].view(torch.uint8).fill_(255)


@pytest.mark.parametrize("paged", [False, True])
def test_decode_reads_only_written_memory(paged):
    """Caches whose memory starts as NaN bytes: 4..8 outliers per token with rank
    <= 4 (Rf rows of four floats) take the decoder's eight-rank outlier path,
    which must not read past a row's own Rf floats (past channel 127's row lies
    the next block, never written). Attention against the oracle."""
    B, H, Hq, dtype, n0, n_b = 2, 2, 4, "f16", 150, 16
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.05, rank=4, buffer_len=n_b, buffer_rank=2,
                         power_iters=3, seed=3)
    op = oracle_params(p)
    xk = seeded_kv(51, 1, (B, H, n0, 128), dtype, channel_scale=True)
    xv = seeded_kv(51, 2, (B, H, n0, 128), dtype)
    if paged:
        kc = gear.PagedCache(p, B, H, 64, 16, 6, 6, TORCH_DT[dtype])
        vc = gear.PagedCache(p, B, H, 64, 16, 6, 6, TORCH_DT[dtype])
    else:
        kc = gear.Cache(p, B, H, 320, 6, TORCH_DT[dtype])
        vc = gear.Cache(p, B, H, 320, 6, TORCH_DT[dtype])
    _poison(kc)
    _poison(vc)
    if paged:
        kc.encode_rows([0, 1], to_dev(xk, dtype))
        vc.encode_rows([0, 1], to_dev(xv, dtype))
    else:
        kc.encode(to_dev(xk, dtype))
        vc.encode(to_dev(xv, dtype))
    ok, ov = oracle.Cache(op, B, H, 128), oracle.Cache(op, B, H, 128)
    ok.encode(xk)
    ov.encode(xv)
    for i in range(n_b + 3):   # one flush
        rk = seeded_kv(900 + i, 3, (B, H, 128), dtype)
        rv = seeded_kv(900 + i, 4, (B, H, 128), dtype)
        if paged:
            gear.append_rows(kc, vc, [0, 1], to_dev(rk, dtype), to_dev(rv, dtype))
        else:
            gear.append_buffer(kc, vc, to_dev(rk, dtype), to_dev(rv, dtype))
        ok.append(rk)
        ov.append(rv)
    # the case that matters is there: channel 127 is an outlier in the last block
    assert any((u.oidx == 127).any() for u in ok.blocks[-1] + ov.blocks[-1])
    q = seeded_kv(71, 5, (B, Hq, 128), dtype)
    out = gear.decode_attn(kc, vc, to_dev(q, dtype), TAU, out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    od = oracle.decode_attn(ok, ov, q, TAU)
    vmax = np.abs(ov.dense()).max()
    assert np.isfinite(out).all()
    assert np.abs(out - od).max() <= 1e-3 * vmax


@pytest.mark.parametrize("paged", [False, True])
def test_workspace_reads_only_what_it_wrote(paged):
    """The shared workspace filled with 0xFF bytes (NaN) before every encode,
    flush and decode: the encoder's Gram partials and Z slabs, the staging
    copies of the paged layout and the decode partials must all be written
    before they are read."""
    B, H, Hq, dtype, n0, n_b = 2, 2, 4, "bf16", 300, 20
    p = gear.make_params(bits=2, group_size=32, outlier_frac=0.05, rank=8, buffer_len=n_b, buffer_rank=2,
                         power_iters=3, seed=13)
    op = oracle_params(p)
    xk = seeded_kv(61, 1, (B, H, n0, 128), dtype, channel_scale=True)
    xv = seeded_kv(61, 2, (B, H, n0, 128), dtype)

    def poison():
        torch.cuda.synchronize()
        ws = gear.gear._ws
        ws.get(64 << 20, "cuda")
        ws.buf.fill_(255)

    if paged:
        kc = gear.PagedCache(p, B, H, 128, 16, 4, 4, TORCH_DT[dtype])
        vc = gear.PagedCache(p, B, H, 128, 16, 4, 4, TORCH_DT[dtype])
        poison()
        kc.encode_rows([0, 1], to_dev(xk, dtype))
        poison()
        vc.encode_rows([0, 1], to_dev(xv, dtype))
    else:
        kc = gear.Cache(p, B, H, 400, 4, TORCH_DT[dtype])
        vc = gear.Cache(p, B, H, 400, 4, TORCH_DT[dtype])
        poison()
        kc.encode(to_dev(xk, dtype))
        poison()
        vc.encode(to_dev(xv, dtype))
    ok, ov = oracle.Cache(op, B, H, 128), oracle.Cache(op, B, H, 128)
    ok.encode(xk)
    ov.encode(xv)
    for i in range(n_b + 2):   # one flush
        rk = seeded_kv(700 + i, 3, (B, H, 128), dtype)
        rv = seeded_kv(700 + i, 4, (B, H, 128), dtype)
        poison()
        if paged:
            gear.append_rows(kc, vc, [0, 1], to_dev(rk, dtype), to_dev(rv, dtype))
        else:
            gear.append_buffer(kc, vc, to_dev(rk, dtype), to_dev(rv, dtype))
        ok.append(rk)
        ov.append(rv)
    q = seeded_kv(81, 5, (B, Hq, 128), dtype)
    poison()
    out = gear.decode_attn(kc, vc, to_dev(q, dtype), TAU, out_dtype=torch.float32).cpu().numpy()
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    od = oracle.decode_attn(ok, ov, q, TAU)
    assert np.isfinite(out).all()
    assert np.abs(out - od).max() <= _tol_out(dtype) * np.abs(ov.dense()).max()
