"""Host-side checks of the C ABI (no GPU): the library loads and exports every
function include/gear.h declares, the ctypes structs match the C layout, and
invalid arguments are rejected on the host before anything is enqueued."""
import ctypes
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gear.h")


@pytest.fixture(scope="module")
def gear():
    from kv_cache_compression_gear_b200 import build
    build.build()
    import kv_cache_compression_gear_b200 as g
    return g


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(gear_[a-z_]+)\s*\(", src)))


def test_exports_every_declared_function(gear):
    names = declared_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(gear.lib, n), n
    out = subprocess.run(["nm", "-D", "--defined-only", gear.gear.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (gear_\w+)", out))
    assert set(names) <= exported


def test_struct_layout_matches_c(gear):
    prog = r'''
#include <stdio.h>
#include <stddef.h>
#include "gear.h"
int main(void) {
  printf("%zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(gear_params), sizeof(gear_cache),
         offsetof(gear_cache, p), offsetof(gear_cache, codes), offsetof(gear_cache, buf),
         offsetof(gear_cache, n_comp), offsetof(gear_params, seed), offsetof(gear_cache, page_tokens),
         offsetof(gear_cache, table), offsetof(gear_cache, host));
  return 0;
}'''
    with tempfile.TemporaryDirectory() as td:
        c = os.path.join(td, "t.c")
        open(c, "w").write(prog)
        exe = os.path.join(td, "t")
        subprocess.check_call(["gcc", "-I", os.path.join(ROOT, "include"), c, "-o", exe])
        vals = [int(v) for v in subprocess.check_output([exe]).split()]
    G, P = gear.GearCacheStruct, gear.GearParams
    assert vals == [ctypes.sizeof(P), ctypes.sizeof(G), G.p.offset, G.codes.offset, G.buf.offset,
                    G.n_comp.offset, P.seed.offset, G.page_tokens.offset, G.table.offset, G.host.offset]


def test_num_outliers_and_validation(gear):
    L = gear.lib
    assert L.gear_num_outliers(ctypes.c_float(0.02), 128) == 3
    assert L.gear_num_outliers(ctypes.c_float(0.05), 128) == 7
    assert L.gear_num_outliers(ctypes.c_float(0.0), 128) == 0
    ok = gear.make_params()
    assert L.gear_validate_params(ctypes.byref(ok), 128) == 0
    bad = [dict(bits=3), dict(group_size=48), dict(group_size=8, bits=2), dict(outlier_frac=-0.1),
           dict(outlier_frac=0.6), dict(rank=-1), dict(rank=17), dict(power_iters=0), dict(buffer_len=0),
           dict(buffer_rank=21)]
    for kw in bad:
        p = gear.make_params(**kw)
        assert L.gear_validate_params(ctypes.byref(p), 128) == gear.gear.GEAR_ERR_INVALID_ARG, kw
    assert L.gear_validate_params(ctypes.byref(ok), 64) == gear.gear.GEAR_ERR_UNSUPPORTED
    p = gear.make_params(group_size=16, bits=2)   # valid, but groups below 32 channels are not implemented
    assert L.gear_validate_params(ctypes.byref(p), 128) == gear.gear.GEAR_ERR_UNSUPPORTED
    p = gear.make_params(outlier_frac=0.2)   # k = 26 > 16
    assert L.gear_validate_params(ctypes.byref(p), 128) == gear.gear.GEAR_ERR_UNSUPPORTED
    assert L.gear_validate_params(None, 128) == gear.gear.GEAR_ERR_INVALID_ARG


def test_cache_layout_and_host_errors(gear):
    L = gear.lib
    p = gear.make_params()
    nbytes = L.gear_cache_bytes(ctypes.byref(p), 1, 32, 128, 4096, 1, 0)
    # codes 64 B + meta 16 B + 3 idx + 3 fp16 values + 4 fp16 L per token
    per_tok = 64 + 16 + 3 + 6 + 8
    assert per_tok * 32 * 4096 <= nbytes <= per_tok * 32 * 4096 + 32 * 20 * 256 + 32 * 4 * 512 + 8 * 256
    c = gear.GearCacheStruct()
    fake = ctypes.c_void_p(1 << 40)  # never dereferenced on the host
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(p), 1, 32, 128, 4096, 1, 0, fake, nbytes - 1) == \
        gear.gear.GEAR_ERR_CAPACITY
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(p), 1, 32, 128, 4096, 1, 0,
                             ctypes.c_void_p((1 << 40) + 8), nbytes) == gear.gear.GEAR_ERR_INVALID_ARG
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(p), 1, 32, 128, 4096, 1, 0, fake, nbytes) == 0
    assert (c.k, c.G, c.W, c.r_max) == (3, 2, 16, 4)
    assert c.codes == 1 << 40 and c.n_comp == 0
    offs = [c.codes, c.meta, c.oidx, c.oval, c.lfac, c.rfac, c.buf]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert c.buf + 32 * 20 * 128 * 2 <= (1 << 40) + nbytes
    # argument errors return before touching the device
    E = gear.gear
    assert L.gear_encode(ctypes.byref(c), None, 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode(ctypes.byref(c), ctypes.c_void_p(4096 + 8), 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode(ctypes.byref(c), ctypes.c_void_p(4096), 0, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode(ctypes.byref(c), ctypes.c_void_p(4096), 5000, None, 0, None) == E.GEAR_ERR_CAPACITY
    assert L.gear_encode(ctypes.byref(c), ctypes.c_void_p(4096), 2, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_decode_attn(ctypes.byref(c), ctypes.byref(c), ctypes.c_void_p(4096), 32, ctypes.c_float(0.1),
                              ctypes.c_void_p(4096), 0, None, 0, None) == E.GEAR_ERR_INVALID_ARG  # empty cache
    # reset empties the host counters and touches nothing else
    c.n_comp, c.n_buf, c.n_blk, c.blk0_len, c.blk0_rank = 4096, 3, 1, 4096, 4
    before = (c.codes, c.meta, c.buf, c.k, c.W)
    assert L.gear_cache_reset(ctypes.byref(c)) == 0
    assert (c.n_comp, c.n_buf, c.n_blk, c.blk0_len, c.blk0_rank) == (0, 0, 0, 0, 0)
    assert (c.codes, c.meta, c.buf, c.k, c.W) == before
    assert L.gear_cache_reset(None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_decode_attn_ragged(ctypes.byref(c), ctypes.byref(c), ctypes.c_void_p(4096), 32, ctypes.c_float(0.1),
                                     ctypes.c_void_p(4096), 0, None, ctypes.c_void_p(4096), 1 << 20,
                                     None) == E.GEAR_ERR_INVALID_ARG   # no prefill lengths
    assert L.gear_decode_dense(ctypes.byref(c), None, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_selftest_wait_timeout(0, None) == E.GEAR_ERR_INVALID_ARG   # rejected before any launch
    assert L.gear_status_string(6) == b"workspace missing or too small"
    assert L.gear_version() == b"0.1.0"


def test_f16_metadata_layout_and_errors(gear):
    L, E = gear.lib, gear.gear
    p16 = gear.make_params(meta_f16=True)
    p32 = gear.make_params()
    b16 = L.gear_cache_bytes(ctypes.byref(p16), 1, 32, 128, 4096, 1, 0)
    b32 = L.gear_cache_bytes(ctypes.byref(p32), 1, 32, 128, 4096, 1, 0)
    # two binary16 pairs per token instead of two binary32 pairs: 8 bytes less
    assert b32 - b16 == 8 * 32 * 4096
    assert L.gear_cache_bytes(ctypes.byref(p16), 1, 32, 128, 4096, 1, 1) == 0   # bf16 input
    assert L.gear_cache_bytes(ctypes.byref(p16), 1, 32, 128, 4096, 1, 2) == 0   # f32 input
    c = gear.GearCacheStruct()
    fake = ctypes.c_void_p(1 << 40)
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(p16), 1, 32, 128, 4096, 1, 1, fake, 1 << 30) == \
        E.GEAR_ERR_UNSUPPORTED
    bad = gear.make_params()
    bad.meta_f16 = 2
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(bad), 1, 32, 128, 4096, 1, 0, fake, 1 << 30) == \
        E.GEAR_ERR_INVALID_ARG
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(p16), 1, 32, 128, 4096, 1, 0, fake, b16) == 0
    assert c.p.meta_f16 == 1 and c.oidx - c.meta >= 32 * 4096 * 8


def test_encode_batch_host_errors(gear):
    """gear_encode_batch rejects bad batches before touching the device."""
    L, E = gear.lib, gear.gear
    p = gear.make_params()
    p2 = gear.make_params(bits=2, group_size=32)
    caches = []
    for i, pp in enumerate([p, p, p2]):
        nbytes = L.gear_cache_bytes(ctypes.byref(pp), 1, 4, 128, 1024, 1, 0)
        c = gear.GearCacheStruct()
        assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(pp), 1, 4, 128, 1024, 1, 0,
                                 ctypes.c_void_p((1 << 40) * (i + 1)), nbytes) == 0
        caches.append(c)
    ptrs = lambda cs: (ctypes.c_void_p * len(cs))(*[ctypes.addressof(c) for c in cs])  # noqa: E731
    xs = lambda m: (ctypes.c_void_p * m)(*[4096 * (j + 1) for j in range(m)])  # noqa: E731
    assert L.gear_encode_batch(0, ptrs(caches[:1]), xs(1), 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode_batch(2, ptrs(caches[:2]), xs(2), 0, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    # different parameters, the same cache twice, a misaligned input
    assert L.gear_encode_batch(2, ptrs([caches[0], caches[2]]), xs(2), 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode_batch(2, ptrs([caches[0], caches[0]]), xs(2), 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    bad = (ctypes.c_void_p * 2)(4096, 4096 + 8)
    assert L.gear_encode_batch(2, ptrs(caches[:2]), bad, 10, None, 0, None) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_encode_batch(2, ptrs(caches[:2]), xs(2), 2000, None, 0, None) == E.GEAR_ERR_CAPACITY
    assert L.gear_encode_batch(2, ptrs(caches[:2]), xs(2), 2, None, 0, None) == E.GEAR_ERR_INVALID_ARG  # rank 4 > n
    assert all(c.n_comp == 0 for c in caches)


def test_channel_groups_validation_and_layout(gear):
    """Per-channel key groups (the KIVI-combined quantizer): the buffer holds whole
    groups (at least one), 16-bit caches only, no binary16 metadata; the meta array
    holds one 1 KB slot per token group."""
    L, E = gear.lib, gear.gear
    ok = gear.make_params(group_size=64, buffer_len=128, channel_groups=True)
    assert L.gear_validate_params(ctypes.byref(ok), 128) == 0
    for kw, want in [(dict(buffer_len=32), E.GEAR_ERR_INVALID_ARG),     # shorter than a group
                     (dict(buffer_len=96), E.GEAR_ERR_INVALID_ARG),     # not whole groups
                     (dict(buffer_len=128, meta_f16=True), E.GEAR_ERR_UNSUPPORTED)]:
        bad = gear.make_params(group_size=64, channel_groups=True, **kw)
        assert L.gear_validate_params(ctypes.byref(bad), 128) == want, kw
    bad = gear.make_params(group_size=64, buffer_len=128)
    bad.channel_groups = 2
    assert L.gear_validate_params(ctypes.byref(bad), 128) == E.GEAR_ERR_INVALID_ARG
    assert L.gear_cache_bytes(ctypes.byref(ok), 1, 4, 128, 1000, 2, 2) == 0            # fp32 cache
    c = gear.GearCacheStruct()
    fake = ctypes.c_void_p(1 << 40)
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(ok), 1, 4, 128, 1000, 2, 2, fake, 1 << 30) == \
        E.GEAR_ERR_UNSUPPORTED
    nbytes = L.gear_cache_bytes(ctypes.byref(ok), 1, 4, 128, 1000, 2, 0)
    assert L.gear_cache_init(ctypes.byref(c), ctypes.byref(ok), 1, 4, 128, 1000, 2, 0, fake, nbytes) == 0
    slots = -(-c.n_max // 64) + 1                # n_max is rounded up to 1024
    assert c.n_max == 1024 and c.oidx - c.meta >= 4 * slots * 128 * 8


def test_paged_layout_and_host_errors(gear):
    """The paged layout's sizes, the host state init writes, and the row calls'
    argument errors, all decided on the host. Without a GPU, init's two memsets
    fail (GEAR_ERR_CUDA) after the host state is written."""
    import numpy as np
    L, E = gear.lib, gear.gear
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, buffer_len=20, buffer_rank=2)
    B, H, P, NP, ppr, nblk = 3, 2, 64, 10, 4, 5
    nb = L.gear_paged_cache_bytes(ctypes.byref(p), B, H, 128, P, NP, ppr, nblk, 0)
    per_tok = 64 + 16 + 3 + 6 + 8
    pool = per_tok * NP * H * P
    assert pool <= nb <= pool + B * H * (nblk * 128 * 4 * 4 + 20 * 256) + 12 * 256
    assert L.gear_paged_host_ints(B, ppr, NP) == 3 * B + B * ppr + NP + 1
    for bad in [(B, H, 48, NP, ppr), (B, H, 0, NP, ppr), (0, H, P, NP, ppr), (B, H, P, 0, ppr), (B, H, P, NP, 0)]:
        assert L.gear_paged_cache_bytes(ctypes.byref(p), bad[0], bad[1], 128, bad[2], bad[3], bad[4], nblk, 0) == 0
    # per-channel key groups: the pool loses its per-token meta rows, and each unit
    # keeps ceil(P * ppr / g) + 1 slots of 1 KB; fp32 caches are refused
    pk = gear.make_params(channel_groups=True, buffer_len=64)
    nk = L.gear_paged_cache_bytes(ctypes.byref(pk), B, H, 128, P, NP, ppr, nblk, 0)
    slots = -(-(P * ppr) // 64) + 1
    buf_more = B * H * (64 - 20) * 128 * 2   # the larger buffer (64 tokens, not 20)
    assert abs(nk - (nb - 16 * NP * H * P + B * H * slots * 1024 + buf_more)) <= 4 * 256
    assert L.gear_paged_cache_bytes(ctypes.byref(pk), B, H, 128, P, NP, ppr, nblk, 2) == 0
    nh = L.gear_paged_host_ints(B, ppr, NP)
    host = np.full(nh, 7, dtype=np.int32)
    hp = ctypes.c_void_p(host.ctypes.data)
    c = gear.GearCacheStruct()
    fake = ctypes.c_void_p(1 << 40)
    assert L.gear_paged_cache_init(ctypes.byref(c), ctypes.byref(p), B, H, 128, P, NP, ppr, nblk, 0, fake, nb - 1,
                                   hp, nh, None) == E.GEAR_ERR_CAPACITY
    assert L.gear_paged_cache_init(ctypes.byref(c), ctypes.byref(p), B, H, 128, P, NP, ppr, nblk, 0, fake, nb,
                                   hp, nh - 1, None) == E.GEAR_ERR_CAPACITY
    assert L.gear_paged_cache_init(ctypes.byref(c), ctypes.byref(p), B, H, 128, 40, NP, ppr, nblk, 0, fake, nb,
                                   hp, nh, None) == E.GEAR_ERR_INVALID_ARG
    assert (host == 7).all()   # nothing written on an error
    st = L.gear_paged_cache_init(ctypes.byref(c), ctypes.byref(p), B, H, 128, P, NP, ppr, nblk, 0, fake, nb,
                                 hp, nh, None)
    assert st in (E.GEAR_OK, E.GEAR_ERR_CUDA)
    assert (c.page_tokens, c.num_pages, c.pages_per_row, c.n_max, c.blk0_rank) == (P, NP, ppr, P * ppr, 4)
    offs = [c.codes, c.meta, c.oidx, c.oval, c.lfac, c.rfac, c.buf, c.table, c.rows]
    assert offs == sorted(offs) and all(o % 256 == 0 for o in offs)
    assert c.rows + 3 * B * 4 <= (1 << 40) + nb
    assert (host[:3 * B] == 0).all() and (host[3 * B:3 * B + B * ppr] == -1).all()
    assert list(host[3 * B + B * ppr:-1]) == list(range(NP - 1, -1, -1)) and host[-1] == NP
    # row-call argument errors: returned before anything is enqueued
    rows = (ctypes.c_int32 * 2)(0, 0)
    ws = ctypes.c_void_p(1 << 41)
    kv = ctypes.c_void_p(1 << 42)
    assert L.gear_encode_rows(ctypes.byref(c), rows, 2, kv, 10, ws, 1 << 30, None) == E.GEAR_ERR_INVALID_ARG  # repeated
    rows = (ctypes.c_int32 * 1)(3)
    assert L.gear_encode_rows(ctypes.byref(c), rows, 1, kv, 10, ws, 1 << 30, None) == E.GEAR_ERR_INVALID_ARG  # range
    rows = (ctypes.c_int32 * 1)(1)
    assert L.gear_encode_rows(ctypes.byref(c), rows, 1, kv, 2, ws, 1 << 30, None) == E.GEAR_ERR_INVALID_ARG  # rank > n
    assert L.gear_encode_rows(ctypes.byref(c), rows, 1, kv, P * ppr + 1, ws, 1 << 30, None) == E.GEAR_ERR_CAPACITY
    rows3 = (ctypes.c_int32 * 3)(0, 1, 2)
    assert L.gear_encode_rows(ctypes.byref(c), rows3, 3, kv, 4 * P, ws, 1 << 30, None) == E.GEAR_ERR_CAPACITY  # pages
    assert L.gear_encode_rows(ctypes.byref(c), rows, 1, kv, 100, None, 0, None) == E.GEAR_ERR_WORKSPACE
    assert L.gear_append_rows(ctypes.byref(c), ctypes.byref(c), rows, 1, kv, kv, ws, 1 << 30,
                              None) == E.GEAR_ERR_INVALID_ARG   # one cache as both K and V
    # the contiguous entry points refuse a paged cache
    assert L.gear_encode(ctypes.byref(c), kv, 10, ws, 1 << 30, None) == E.GEAR_ERR_UNSUPPORTED
    assert L.gear_cache_reset(ctypes.byref(c)) == E.GEAR_ERR_UNSUPPORTED
    assert L.gear_decode_dense(ctypes.byref(c), ctypes.c_void_p(1 << 42), None) == E.GEAR_ERR_UNSUPPORTED
    assert (host[:3 * B] == 0).all() and host[-1] == NP   # untouched by the refused calls
