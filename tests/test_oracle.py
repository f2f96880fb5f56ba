"""Pins of the CPU oracle against facts that do not come from the oracle itself:
a published generator test vector, brute force on tiny inputs, the textbook
group-wise quantizer (the s = 0, r = 0 special case), the half-step error
bound, closed forms of power iteration, the Eckart-Young bound and the
truncated SVD, full-rank reconstruction, and textbook softmax attention."""
import os

import numpy as np
import pytest

import oracle
from oracle import Params

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(20240308)


def unpack_codes(codes: np.ndarray, d: int, bits: int) -> np.ndarray:
    """Codes per channel from the packed layout stated in include/gear.h:
    channel c occupies bits [(c*b) % 32, +b) of word (c*b) / 32."""
    c = np.arange(d)
    word = (c * bits) // 32
    sh = (c * bits) % 32
    return (codes[..., word] >> sh.astype(np.uint32)) & np.uint32((1 << bits) - 1)


# ----------------------------------------------------------------- generator
def test_splitmix64_matches_published_test_vector():
    want = [int(l) for l in open(os.path.join(GOLDEN, "splitmix64_seed1234567.txt"))
            if l.strip() and not l.startswith("#")]
    assert oracle.splitmix64_stream(1234567, 5) == want


def test_start_matrix_entries():
    q0 = oracle.start_matrix(1234567, 128, 4)
    outs = oracle.splitmix64_stream(1234567, 128 * 4)
    # entry (i, j) is output i*r + j, top 24 bits mapped to [-1, 1)
    want = np.array([(o >> 40) * 2.0 ** -23 - 1.0 for o in outs]).reshape(128, 4)
    assert np.array_equal(q0, want)
    assert q0.min() >= -1.0 and q0.max() < 1.0
    assert np.all(np.float32(q0) == q0)  # exact in binary32
    # entries are drawn row by row, so a different rank reads the stream differently
    assert not np.array_equal(oracle.start_matrix(1, 128, 2), oracle.start_matrix(1, 128, 4)[:, :2])


# ----------------------------------------------------------------- outliers
@pytest.mark.parametrize("s,d,k", [(0.02, 128, 3), (0.05, 128, 7), (0.0, 128, 0), (0.5, 128, 64),
                                   (1 / 128, 128, 1), (0.02, 64, 2)])
def test_num_outliers(s, d, k):
    assert oracle.num_outliers(s, d) == k


def _brute_outliers(x, k):
    # full sort: |x| descending, then channel ascending
    order = sorted(range(len(x)), key=lambda c: (-abs(float(x[c])), c))
    return np.array(sorted(order[:k]), dtype=np.int32)


@pytest.mark.parametrize("k", [1, 3, 7, 64])
def test_outliers_brute_force(k):
    for trial in range(200):
        if trial % 3 == 0:   # many ties, signed zeros
            x = RNG.integers(-3, 4, size=128).astype(np.float32)
            x[RNG.integers(0, 128, size=5)] = -0.0
        else:
            x = RNG.standard_normal(128).astype(np.float32)
        assert np.array_equal(oracle.select_outliers(x, k), _brute_outliers(x, k))


# ------------------------------------------------------------- quantization
def textbook_groupwise(x, bits, g):
    """Plain per-token group-wise asymmetric min-max quantization (float32)."""
    n, d = x.shape
    L = np.float32(2 ** bits - 1)
    xg = x.reshape(n, d // g, g)
    mn = xg.min(axis=2, keepdims=True)
    mx = xg.max(axis=2, keepdims=True)
    scale = (mx - mn) / L
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(scale > 0, np.rint((xg - mn) / scale), 0).astype(np.float32)
    q = np.clip(q, 0, L)
    return q.reshape(n, d).astype(np.uint32), scale[..., 0], mn[..., 0]


@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32), (8, 32), (4, 32), (2, 128), (8, 128)])
def test_s0_r0_is_textbook_groupwise_quantization(bits, g):
    x = (RNG.standard_normal((64, 128)) * RNG.uniform(0.1, 5, size=(64, 1))).astype(np.float32)
    x[3, :g] = 1.25            # constant group: scale 0
    x[5, 7] = 40.0             # isolated large entry
    p = Params(bits=bits, group_size=g, outlier_frac=0.0, rank=0)
    u = oracle.encode_unit(x, p)
    codes, scale, zero = textbook_groupwise(x, bits, g)
    assert np.array_equal(unpack_codes(u.codes, 128, bits), codes)
    assert np.array_equal(u.scale, scale)
    assert np.array_equal(u.zero, zero)
    dh = oracle.reconstruct_unit(u, p)
    # with r = 0 the reconstruction is code*scale + zero in one fused rounding
    want = np.float32(codes.astype(np.float64).reshape(64, -1, g) * scale[..., None].astype(np.float64)
                      + zero[..., None].astype(np.float64)).reshape(64, 128)
    assert np.array_equal(dh.astype(np.float32), want)


@pytest.mark.parametrize("bits,g,s", [(4, 64, 0.02), (2, 32, 0.05), (8, 64, 0.02), (4, 32, 0.1)])
def test_quantization_invariants(bits, g, s):
    n, d = 300, 128
    x = (RNG.standard_normal((n, d)) * np.exp(RNG.uniform(np.log(0.5), np.log(8), size=(1, d))))
    x = x.astype(np.float16).astype(np.float32)
    p = Params(bits=bits, group_size=g, outlier_frac=s, rank=0)
    u = oracle.encode_unit(x, p)
    k = oracle.num_outliers(s, d)
    L = 2 ** bits - 1
    codes = unpack_codes(u.codes, d, bits)
    out_mask = np.zeros((n, d), bool)
    np.put_along_axis(out_mask, u.oidx.astype(np.int64), True, axis=1)
    assert out_mask.sum() == n * k
    # outliers: exact values, code 0, zero residual
    assert np.array_equal(u.oval, np.take_along_axis(x, u.oidx.astype(np.int64), axis=1))
    assert np.all(codes[out_mask] == 0)
    assert np.all(u.resid[out_mask] == 0)
    assert codes.max() <= L
    G = d // g
    xg = np.where(out_mask, np.nan, x).reshape(n, G, g)
    cg = codes.reshape(n, G, g)
    sc = u.scale.astype(np.float64)
    for t in range(n):
        for j in range(G):
            vals = xg[t, j]
            ok = ~np.isnan(vals)
            if not ok.any():
                assert u.scale[t, j] == 0 and u.zero[t, j] == 0
                continue
            assert u.zero[t, j] == np.nanmin(vals)
            if u.scale[t, j] > 0:
                assert cg[t, j][np.nanargmin(vals)] == 0
                assert cg[t, j][np.nanargmax(vals)] == L
    # half-step bound: |x - dhat| <= scale*(1/2 + L*2^-22) + ulp(dhat)/2 for non-outliers
    dh = oracle.reconstruct_unit(u, p)
    dh32 = dh.astype(np.float32)
    err = np.abs(x.astype(np.float64) - dh32.astype(np.float64))
    bound = np.repeat(sc, g, axis=1) * (0.5 + L * 2.0 ** -22) + 0.5 * np.spacing(np.abs(dh32)).astype(np.float64)
    assert np.all(err[~out_mask] <= bound[~out_mask])
    assert np.array_equal(dh[out_mask], x[out_mask].astype(np.float64))
    # residual definition
    assert np.array_equal(u.resid[~out_mask], (x - dh32)[~out_mask])


def test_signed_zero_minimum_is_stored_as_positive_zero():
    # a group whose minimum is zero, with -0 before +0 and the reverse
    x = np.abs(RNG.standard_normal((2, 128)).astype(np.float32)) + 0.5
    x[0, 3], x[0, 9] = -0.0, 0.0
    x[1, 3], x[1, 9] = 0.0, -0.0
    x[:, 64:] = -0.0                      # second group all -0: scale and zero +0
    p = Params(bits=4, group_size=64, outlier_frac=0.0, rank=0)
    u = oracle.encode_unit(x, p)
    assert np.all(u.zero.view(np.uint32) == 0)
    assert np.all(u.scale[:, 1].view(np.uint32) == 0)
    assert np.all(unpack_codes(u.codes, 128, 4)[:, [3, 9]] == 0)


def test_all_outlier_group():
    # g = 32 with s = 0.5: k = 64 outliers can cover a whole group
    x = np.zeros((1, 128), np.float32)
    x[0, :32] = 100 + np.arange(32)
    x[0, 32:] = RNG.standard_normal(96).astype(np.float32)
    p = Params(bits=4, group_size=32, outlier_frac=0.5, rank=0)
    u = oracle.encode_unit(x, p)
    assert u.scale[0, 0] == 0 and u.zero[0, 0] == 0
    assert set(range(32)).issubset(set(u.oidx[0].tolist()))


# --------------------------------------------------------------- low rank
def test_full_rank_reconstructs_input():
    n, d = 256, 128
    x = RNG.standard_normal((n, d)).astype(np.float32)
    p = Params(bits=2, group_size=32, outlier_frac=0.02, rank=128, power_iters=2, seed=7)
    u = oracle.encode_unit(x, p)
    xh = oracle.reconstruct_unit(u, p)
    assert np.max(np.abs(xh - x)) <= 1e-5 * np.max(np.abs(x))
    # L has orthonormal columns
    assert np.allclose(u.L.T @ u.L, np.eye(128), atol=1e-9)


@pytest.mark.parametrize("r,T", [(1, 1), (4, 3), (8, 3), (4, 5)])
def test_power_iteration_closed_form(r, T):
    n, d = 200, 128
    R = RNG.standard_normal((n, d)).astype(np.float32)
    q0 = oracle.start_matrix(99, d, r)
    L, Rf = oracle.power_iteration(R, r, T, q0)
    R64 = R.astype(np.float64)
    Kr = R64 @ np.linalg.matrix_power(R64.T @ R64, T - 1) @ q0
    Qk, _ = np.linalg.qr(Kr)
    assert np.allclose(L @ L.T, Qk @ Qk.T, atol=1e-9)
    assert np.allclose(Rf, R64.T @ L, atol=1e-9 * np.abs(R64).sum())
    # the QR with positive diagonal is unique: L is that Q factor
    Qs = Qk * np.sign(np.diag(_)).reshape(1, -1)
    assert np.allclose(L, Qs, atol=1e-8)


def test_eckart_young_lower_bound_and_truncated_svd():
    n, d, r = 300, 128, 4
    R = RNG.standard_normal((n, d)).astype(np.float32)
    q0 = oracle.start_matrix(5, d, r)
    L, Rf = oracle.power_iteration(R, r, 3, q0)
    sv = np.linalg.svd(R.astype(np.float64), compute_uv=False)
    err = np.linalg.norm(R - L @ Rf.T)
    assert err >= np.sqrt(np.sum(sv[r:] ** 2)) * (1 - 1e-12)
    # a spectrum with a gap: many iterations converge to the truncated SVD
    U, _, Vt = np.linalg.svd(RNG.standard_normal((n, d)), full_matrices=False)
    s = np.concatenate([[50, 40, 30, 20], np.linspace(2, 1, d - 4)])
    Rg = ((U * s) @ Vt).astype(np.float32)
    L, Rf = oracle.power_iteration(Rg, r, 40, q0)
    Ug, sg, Vg = np.linalg.svd(Rg.astype(np.float64), full_matrices=False)
    best = (Ug[:, :r] * sg[:r]) @ Vg[:r]
    assert np.max(np.abs(L @ Rf.T - best)) <= 1e-6 * np.max(np.abs(best))


def test_rank_deficient_residual_gives_zero_columns():
    n, d = 64, 128
    R = np.zeros((n, d), np.float32)
    R[:, 0] = RNG.standard_normal(n)          # rank 1
    q0 = oracle.start_matrix(3, d, 4)
    L, Rf = oracle.power_iteration(R, 4, 3, q0)
    assert np.allclose(L @ Rf.T, R, atol=1e-12)
    assert np.count_nonzero(np.linalg.norm(L, axis=0)) == 1
    L0, Rf0 = oracle.power_iteration(np.zeros((n, d), np.float32), 4, 3, q0)
    assert not L0.any() and not Rf0.any()


def test_low_rank_reduces_residual():
    x = (RNG.standard_normal((512, 128)) * np.linspace(0.5, 8, 128)).astype(np.float32)
    p0 = Params(bits=4, group_size=64, outlier_frac=0.02, rank=0)
    p4 = Params(bits=4, group_size=64, outlier_frac=0.02, rank=4, power_iters=3, seed=11)
    e0 = np.linalg.norm(oracle.reconstruct_unit(oracle.encode_unit(x, p0), p0) - x)
    e4 = np.linalg.norm(oracle.reconstruct_unit(oracle.encode_unit(x, p4), p4) - x)
    assert e4 < e0


# ---------------------------------------------------------------- attention
def test_attention_is_textbook_softmax():
    n, d = 77, 128
    q = RNG.standard_normal(d)
    K = RNG.standard_normal((n, d))
    V = RNG.standard_normal((n, d))
    tau = 1 / np.sqrt(d)
    s = tau * (K @ q)
    w = np.exp(s - s.max())
    w /= w.sum()
    assert np.allclose(oracle.attention(q, K, V, tau), w @ V, rtol=1e-12, atol=1e-12)


def test_cache_attention_buffer_only_and_8bit_closeness():
    B, H, Hq, d = 1, 2, 4, 128
    p = Params(bits=8, group_size=32, outlier_frac=0.0, rank=0, buffer_len=5)
    kc = oracle.Cache(p, B, H, d)
    vc = oracle.Cache(p, B, H, d)
    rows_k = [RNG.standard_normal((B, H, d)).astype(np.float16).astype(np.float32) for _ in range(4)]
    rows_v = [RNG.standard_normal((B, H, d)).astype(np.float16).astype(np.float32) for _ in range(4)]
    for a, b in zip(rows_k, rows_v):
        kc.append(a)
        vc.append(b)
    q = RNG.standard_normal((B, Hq, d))
    out = oracle.decode_attn(kc, vc, q, 0.1)
    K = np.stack(rows_k, 2).astype(np.float64)
    V = np.stack(rows_v, 2).astype(np.float64)
    for j in range(Hq):
        h = j // 2
        s = 0.1 * K[0, h] @ q[0, j]
        w = np.exp(s - s.max())
        w /= w.sum()
        assert np.allclose(out[0, j], w @ V[0, h], rtol=1e-12, atol=1e-12)
    # 8-bit, s = 0, r = 0 compressed cache stays close to attention on the raw values
    X = RNG.standard_normal((B, H, 64, d)).astype(np.float32)
    Y = RNG.standard_normal((B, H, 64, d)).astype(np.float32)
    kc = oracle.Cache(p, B, H, d)
    vc = oracle.Cache(p, B, H, d)
    kc.encode(X)
    vc.encode(Y)
    out = oracle.decode_attn(kc, vc, q, 1 / np.sqrt(d))
    for j in range(Hq):
        ref = oracle.attention(q[0, j], X[0, j // 2], Y[0, j // 2], 1 / np.sqrt(d))
        assert np.max(np.abs(out[0, j] - ref)) < 2e-2


def test_append_flush_protocol():
    B, H, d = 1, 3, 128
    p = Params(bits=4, group_size=64, outlier_frac=0.02, rank=4, buffer_len=4, buffer_rank=2, seed=9)
    kc = oracle.Cache(p, B, H, d)
    X0 = RNG.standard_normal((B, H, 40, d)).astype(np.float32)
    kc.encode(X0)
    rows = [RNG.standard_normal((B, H, d)).astype(np.float32) for _ in range(11)]
    for m, row in enumerate(rows, start=1):
        kc.append(row)
        assert kc.n_comp + len(kc.buffer) == 40 + m
        # lazy flush: a full buffer persists until the next append
        assert 1 <= len(kc.buffer) <= 4
    assert len(kc.blocks) == 3 and kc.n_comp == 48 and len(kc.buffer) == 3
    # a flushed block equals a standalone encode of those tokens with the buffer rank
    blk = np.stack(rows[0:4], 2)
    for u in range(H):
        alone = oracle.encode_unit(blk[0, u], p, rank=2)
        got = kc.blocks[1][u]
        assert np.array_equal(got.codes, alone.codes) and np.array_equal(got.oidx, alone.oidx)
        assert np.array_equal(got.L, alone.L) and got.rank == 2


# ------------------------------------------------ byte-lean (binary16) metadata
@pytest.mark.parametrize("bits,g", [(4, 64), (2, 32), (8, 128)])
def test_f16_metadata_is_textbook_quantization_against_rounded_metadata(bits, g):
    """With scale and zero stored as binary16, s = r = 0 is the textbook quantizer
    run against the rounded metadata (numpy's float16 rounding, independent of
    the C compiler's)."""
    x = (RNG.standard_normal((48, 128)) * RNG.uniform(0.05, 30, size=(48, 1))).astype(np.float16).astype(np.float32)
    x[2, :g] = 0.5             # constant group: scale 0
    p = Params(bits=bits, group_size=g, outlier_frac=0.0, rank=0, meta_f16=True)
    u = oracle.encode_unit(x, p)
    L = 2 ** bits - 1
    xg = x.reshape(48, -1, g)
    mn = xg.min(axis=2, keepdims=True)
    mx = xg.max(axis=2, keepdims=True)
    scale = ((mx - mn) / np.float32(L)).astype(np.float32).astype(np.float16).astype(np.float32)
    zero = mn.astype(np.float16).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(scale > 0, np.rint((xg - zero) / scale), 0).astype(np.float32)
    codes = np.clip(q, 0, L).reshape(48, 128).astype(np.uint32)
    assert np.array_equal(unpack_codes(u.codes, 128, bits), codes)
    assert np.array_equal(u.scale, scale[..., 0])
    assert np.array_equal(u.zero, zero[..., 0])
    # binary16 inputs: the zero point (a group minimum) is stored exactly
    assert np.array_equal(u.zero, mn[..., 0])


@pytest.mark.parametrize("bits,g,s", [(4, 64, 0.02), (2, 32, 0.05)])
def test_f16_metadata_error_bound(bits, g, s):
    """Half a step of the stored scale, plus what rounding the scale moves the
    top of the range by (the code there is clamped)."""
    n, d = 200, 128
    x = (RNG.standard_normal((n, d)) * np.exp(RNG.uniform(np.log(0.5), np.log(8), size=(1, d))))
    x = x.astype(np.float16).astype(np.float32)
    p = Params(bits=bits, group_size=g, outlier_frac=s, rank=0, meta_f16=True)
    u = oracle.encode_unit(x, p)
    L = 2 ** bits - 1
    out_mask = np.zeros((n, d), bool)
    np.put_along_axis(out_mask, u.oidx.astype(np.int64), True, axis=1)
    G = d // g
    xg = np.where(out_mask, np.nan, x).reshape(n, G, g).astype(np.float64)
    exact = (np.nanmax(xg, axis=2) - np.nanmin(xg, axis=2)) / L
    sc = u.scale.astype(np.float64)
    # binary16 rounding (half an ulp, 2^-11 relative; 2^-25 absolute below the normal range) of a binary32 value
    assert np.all(np.abs(sc - exact) <= exact * (2.0 ** -11 + 2.0 ** -22) + 2.0 ** -25)
    dh = oracle.reconstruct_unit(u, p).astype(np.float32).astype(np.float64)
    err = np.abs(x.astype(np.float64) - dh)
    bound = np.repeat(sc * (0.5 + L * 2.0 ** -22) + L * np.abs(sc - exact), g, axis=1) \
        + 0.5 * np.spacing(np.abs(dh.astype(np.float32))).astype(np.float64)
    assert np.all(err[~out_mask] <= bound[~out_mask])
    assert np.array_equal(dh[out_mask], x[out_mask].astype(np.float64))


def test_ragged_prefill_equals_unpadded_cache():
    """With r = 0 every token's reconstruction depends on that token alone, so
    attention over a right-padded prefill with the padding masked must equal
    attention over a cache built from the real tokens only (same appends). This
    ties the masked path to an independently built cache, not to itself."""
    rng = np.random.default_rng(17)
    B, H, Hq, n0, d, nb = 3, 2, 4, 40, 128, 5
    p = Params(bits=4, group_size=64, outlier_frac=0.05, rank=0, power_iters=1, buffer_len=nb, buffer_rank=0,
               seed=3)
    xk = rng.standard_normal((B, H, n0, d)).astype(np.float32)
    xv = rng.standard_normal((B, H, n0, d)).astype(np.float32)
    rows_k = [rng.standard_normal((B, H, d)).astype(np.float32) for _ in range(7)]
    rows_v = [rng.standard_normal((B, H, d)).astype(np.float32) for _ in range(7)]
    q = rng.standard_normal((B, Hq, d))
    plen = [17, 40, 1]
    pk, pv = oracle.Cache(p, B, H, d), oracle.Cache(p, B, H, d)
    pk.encode(xk)
    pv.encode(xv)
    for rk, rv in zip(rows_k, rows_v):
        pk.append(rk)
        pv.append(rv)
    got = oracle.decode_attn(pk, pv, q, 0.09, prefill_len=plen)
    for b in range(B):
        sk, sv = oracle.Cache(p, 1, H, d), oracle.Cache(p, 1, H, d)
        sk.encode(xk[b:b + 1, :, :plen[b]])
        sv.encode(xv[b:b + 1, :, :plen[b]])
        for rk, rv in zip(rows_k, rows_v):
            sk.append(rk[b:b + 1])
            sv.append(rv[b:b + 1])
        want = oracle.decode_attn(sk, sv, q[b:b + 1], 0.09)
        assert np.array_equal(got[b], want[0]), b
    # a full-length prefill is the plain decode
    np.testing.assert_array_equal(oracle.decode_attn(pk, pv, q, 0.09, prefill_len=[n0] * B),
                                  oracle.decode_attn(pk, pv, q, 0.09))


def test_ragged_prefill_all_padding():
    """Prefill length 0: only appended tokens count; with none, the output is 0."""
    rng = np.random.default_rng(5)
    B, H, d = 2, 1, 128
    p = Params(bits=4, group_size=64, outlier_frac=0.02, rank=2, power_iters=2, buffer_len=4, buffer_rank=1, seed=1)
    x = rng.standard_normal((B, H, 30, d)).astype(np.float32)
    q = rng.standard_normal((B, H, d))
    kc, vc = oracle.Cache(p, B, H, d), oracle.Cache(p, B, H, d)
    kc.encode(x)
    vc.encode(-x)
    out = oracle.decode_attn(kc, vc, q, 0.1, prefill_len=[0, 30])
    assert not out[0].any()
    np.testing.assert_array_equal(out[1], oracle.decode_attn(kc, vc, q, 0.1)[1])
    row = rng.standard_normal((B, H, d)).astype(np.float32)
    kc.append(row)
    vc.append(2 * row)
    out = oracle.decode_attn(kc, vc, q, 0.1, prefill_len=[0, 0])
    np.testing.assert_allclose(out[:, 0], 2 * row[:, 0], rtol=0, atol=1e-12)   # one real token: its value


# ------------------------------------ KIVI-combined keys: per-channel token groups
def textbook_channel_groups(x: np.ndarray, bits: int, g: int):
    """Independent restatement: per channel, min-max over each group of g
    consecutive tokens (last group shorter), binary32 arithmetic, ties to even."""
    n, d = x.shape
    L = np.float32(2 ** bits - 1)
    codes = np.zeros((n, d), np.uint32)
    ng = (n + g - 1) // g
    scale = np.zeros((ng, d), np.float32)
    zero = np.zeros((ng, d), np.float32)
    for j in range(ng):
        xs = x[j * g:(j + 1) * g]
        mn = xs.min(axis=0) + np.float32(0.0)
        mx = xs.max(axis=0) + np.float32(0.0)
        sc = (mx - mn) / L
        with np.errstate(divide="ignore", invalid="ignore"):
            q = np.where(sc > 0, np.rint((xs - mn) / sc), 0).astype(np.float32)
        codes[j * g:(j + 1) * g] = np.clip(q, 0, L).astype(np.uint32)
        scale[j], zero[j] = sc, mn
    return codes, scale, zero


@pytest.mark.parametrize("bits,g,n", [(2, 32, 128), (4, 64, 200), (8, 32, 77), (4, 128, 256), (2, 64, 1)])
def test_channel_groups_s0_r0_is_textbook_per_channel_quantization(bits, g, n):
    x = (RNG.standard_normal((n, 128)) * np.exp(RNG.uniform(-1, 2, size=(1, 128)))).astype(np.float32)
    x[:, 5] = 0.75              # a constant channel: scale 0 in every group
    p = Params(bits=bits, group_size=g, outlier_frac=0.0, rank=0, channel_groups=True)
    u = oracle.encode_unit(x, p)
    codes, scale, zero = textbook_channel_groups(x, bits, g)
    assert np.array_equal(unpack_codes(u.codes, 128, bits), codes)
    assert np.array_equal(u.scale, scale) and np.array_equal(u.zero, zero)
    assert u.scale.shape == ((n + g - 1) // g, 128)
    dh = oracle.reconstruct_unit(u, p).astype(np.float32)
    grp = np.arange(n) // g
    want = np.float32(codes.astype(np.float64) * scale[grp].astype(np.float64) + zero[grp].astype(np.float64))
    assert np.array_equal(dh, want)


@pytest.mark.parametrize("bits,g", [(2, 32), (4, 64), (8, 32)])
def test_channel_groups_equal_per_token_quantizer_of_the_transpose(bits, g):
    """Per-channel groups of g tokens of X are per-token groups of g entries of X^T:
    the per-token quantizer (pinned above against the textbook) on the rows of X^T
    must give the same codes, scales and zero points."""
    n = 4 * g
    x = (RNG.standard_normal((n, 128)) * 3).astype(np.float16).astype(np.float32)
    u = oracle.encode_unit(x, Params(bits=bits, group_size=g, outlier_frac=0.0, rank=0, channel_groups=True))
    codes = unpack_codes(u.codes, 128, bits)
    for c in range(0, 128, 13):
        tc, ts, tz, _, _ = oracle.quantize_token(np.ascontiguousarray(x[:, c]), bits, g, np.zeros(0, np.int32))
        assert np.array_equal(unpack_codes(tc, n, bits), codes[:, c])
        assert np.array_equal(ts, u.scale[:, c]) and np.array_equal(tz, u.zero[:, c])


@pytest.mark.parametrize("bits,g,s,n", [(2, 32, 0.05, 160), (4, 64, 0.02, 300), (4, 32, 0.1, 45)])
def test_channel_groups_invariants(bits, g, s, n):
    d = 128
    x = (RNG.standard_normal((n, d)) * np.exp(RNG.uniform(np.log(0.5), np.log(8), size=(1, d))))
    x = x.astype(np.float16).astype(np.float32)
    p = Params(bits=bits, group_size=g, outlier_frac=s, rank=0, channel_groups=True)
    u = oracle.encode_unit(x, p)
    L = 2 ** bits - 1
    codes = unpack_codes(u.codes, d, bits)
    out_mask = np.zeros((n, d), bool)
    np.put_along_axis(out_mask, u.oidx.astype(np.int64), True, axis=1)
    # outliers per token as in GEAR: the same selection, exact values, code 0, zero residual
    for t in range(0, n, 7):
        assert np.array_equal(u.oidx[t], oracle.select_outliers(x[t], oracle.num_outliers(s, d)))
    assert np.array_equal(u.oval, np.take_along_axis(x, u.oidx.astype(np.int64), axis=1))
    assert np.all(codes[out_mask] == 0) and np.all(u.resid[out_mask] == 0)
    grp = np.arange(n) // g
    for j in range((n + g - 1) // g):
        rows = grp == j
        for c in range(d):
            vals = x[rows, c][~out_mask[rows, c]]
            if vals.size == 0:
                assert u.scale[j, c] == 0 and u.zero[j, c] == 0
                continue
            assert u.zero[j, c] == vals.min() + np.float32(0)
            if u.scale[j, c] > 0:
                cc = codes[rows, c][~out_mask[rows, c]]
                assert cc[np.argmin(vals)] == 0 and cc[np.argmax(vals)] == L
    dh = oracle.reconstruct_unit(u, p).astype(np.float32)
    err = np.abs(x.astype(np.float64) - dh.astype(np.float64))
    bound = u.scale[grp].astype(np.float64) * (0.5 + L * 2.0 ** -22) + 0.5 * np.spacing(np.abs(dh)).astype(np.float64)
    assert np.all(err[~out_mask] <= bound[~out_mask])
    assert np.array_equal(dh[out_mask], x[out_mask])


def test_channel_groups_flush_protocol_and_low_rank():
    """A buffer of n_b = 2g tokens flushes as whole groups; the flushed block equals a
    standalone per-channel encode, and attention over the cache is textbook attention
    over the reconstruction."""
    B, H, d, g = 1, 2, 128, 32
    p = Params(bits=2, group_size=g, outlier_frac=0.05, rank=4, buffer_len=2 * g, buffer_rank=2, seed=5,
               channel_groups=True)
    kc = oracle.Cache(p, B, H, d)
    X0 = RNG.standard_normal((B, H, 70, d)).astype(np.float32)   # block 0 ends in a partial group
    kc.encode(X0)
    assert kc.blocks[0][0].scale.shape == (3, d)
    rows = [RNG.standard_normal((B, H, d)).astype(np.float32) for _ in range(2 * g + 3)]
    for row in rows:
        kc.append(row)
    assert kc.n_comp == 70 + 2 * g and len(kc.buffer) == 3
    blk = np.stack(rows[:2 * g], 2)
    for h in range(H):
        alone = oracle.encode_unit(blk[0, h], p, rank=2)
        got = kc.blocks[1][h]
        assert np.array_equal(got.codes, alone.codes) and np.array_equal(got.scale, alone.scale)
        assert got.scale.shape == (2, d)
    # the low-rank factors shrink the residual of the key block
    u = kc.blocks[0][0]
    rec = oracle.reconstruct_unit(u, p)
    nol = oracle.reconstruct_unit(oracle.Unit(u.codes, u.scale, u.zero, u.oidx, u.oval, u.resid,
                                              u.L[:, :0], u.Rf[:, :0], 0), p)
    assert np.linalg.norm(rec - X0[0, 0]) < np.linalg.norm(nol - X0[0, 0])
