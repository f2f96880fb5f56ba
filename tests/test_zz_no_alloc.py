"""The decode entry point that allocates nothing, for callers that cannot call
cudaMalloc (a plugin in a framework that owns all device memory, a decode loop
with a memory budget fixed at start-up). It must give the same attention output
as gear_decode_attn, within the tolerance of the parity tests, on consecutive
calls that share its built-in scratch array, and must refuse problems whose
partial results exceed that array. The file is named to be collected last."""
import ctypes
import math

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


def _cp(c):
    return ctypes.byref(c.c)


@pytest.mark.parametrize("B,H,Hq,n0", [(2, 4, 8, 700), (1, 2, 16, 500)])   # 2 and 8 query heads per kv head
def test_noalloc_decode_matches_workspace_decode(B, H, Hq, n0):
    import kv_cache_compression_gear_b200 as gear
    from kv_cache_compression_gear_b200 import gear as G
    from tests.gpu_helpers import seeded_kv, to_dev

    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, buffer_len=5, buffer_rank=2, seed=31)
    kc = gear.Cache(p, B, H, n0 + 16, 4, torch.float16)
    vc = gear.Cache(p, B, H, n0 + 16, 4, torch.float16)
    kc.encode(to_dev(seeded_kv(5, 1, (B, H, n0, 128), "f16", channel_scale=True), "f16"))
    vc.encode(to_dev(seeded_kv(5, 2, (B, H, n0, 128), "f16"), "f16"))
    for i in range(7):  # one flush, two tokens left in the buffer
        gear.append_buffer(kc, vc, to_dev(seeded_kv(50 + i, 3, (B, H, 128), "f16"), "f16"),
                           to_dev(seeded_kv(50 + i, 4, (B, H, 128), "f16"), "f16"))
    assert G.lib.gear_decode_workspace_bytes(_cp(kc), _cp(vc), Hq) <= (4 << 20)   # fits the scratch array
    vmax = float(vc.dense().abs().max())
    tau = 1.0 / math.sqrt(128)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):   # two calls in a row share the scratch array
        q = to_dev(seeded_kv(70 + call, 5, (B, Hq, 128), "f16"), "f16")
        ref = gear.decode_attn(kc, vc, q, tau, out_dtype=torch.float32)
        out = torch.full((B, Hq, 128), float("nan"), dtype=torch.float32, device="cuda")
        st = G.lib.gear_decode_attn_noalloc(_cp(kc), _cp(vc), ctypes.c_void_p(q.data_ptr()), Hq,
                                            ctypes.c_float(tau), ctypes.c_void_p(out.data_ptr()), G.GEAR_F32,
                                            stream)
        assert st == G.GEAR_OK, G.status_string(st)
        torch.cuda.synchronize()
        err = float((out - ref).abs().max())
        assert err <= 1e-3 * vmax, f"call {call}: {err:.3e} > {1e-3 * vmax:.3e}"
    assert gear.device_status() == 0


def test_noalloc_decode_rejects_oversized_problem():
    import kv_cache_compression_gear_b200 as gear
    from kv_cache_compression_gear_b200 import gear as G

    # 32 x 256 query rows (8 query heads per kv head) need 8192 * 520 B of
    # partials, more than the 4 MiB scratch array: the call must refuse
    B, H, Hq, n = 32, 32, 256, 256
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=0, buffer_len=4, buffer_rank=0)
    kc = gear.Cache(p, B, H, n, 2, torch.float16)
    vc = gear.Cache(p, B, H, n, 2, torch.float16)
    x = torch.zeros((B, H, n, 128), dtype=torch.float16, device="cuda")
    kc.encode(x)
    vc.encode(x)
    need = G.lib.gear_decode_workspace_bytes(_cp(kc), _cp(vc), Hq)
    assert need > (4 << 20)
    q = torch.zeros((B, Hq, 128), dtype=torch.float16, device="cuda")
    out = torch.zeros_like(q)
    st = G.lib.gear_decode_attn_noalloc(_cp(kc), _cp(vc), ctypes.c_void_p(q.data_ptr()), Hq, ctypes.c_float(0.1),
                                        ctypes.c_void_p(out.data_ptr()), G.GEAR_F16, None)
    assert st == G.GEAR_ERR_WORKSPACE
