"""Failure detection on the GPU without a fault: a bounded wait that nothing
completes runs out, the kernel records GEAR_ERR_TIMEOUT in the device error word
and returns, and the context stays usable for the codec afterwards."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.gpu_helpers import TORCH_DT, oracle_params, seeded_kv, to_dev

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import kv_cache_compression_gear_b200 as gear
    from kv_cache_compression_gear_b200 import gear as G
else:
    gear = G = None


def test_bounded_wait_reports_timeout_and_context_survives():
    L = gear.lib
    assert gear.device_status() == 0
    assert L.gear_selftest_wait_timeout(0, None) == G.GEAR_ERR_INVALID_ARG
    assert L.gear_selftest_wait_timeout(1000001, None) == G.GEAR_ERR_INVALID_ARG
    assert L.gear_selftest_wait_timeout(20000, None) == G.GEAR_OK   # 20 ms
    torch.cuda.synchronize()
    assert gear.device_status() == G.GEAR_ERR_TIMEOUT
    assert gear.device_status() == 0   # the read clears the word

    # the same context still encodes and decodes correctly
    p = gear.make_params(bits=4, group_size=64, outlier_frac=0.02, rank=4, power_iters=3, buffer_len=20,
                         buffer_rank=2, seed=5)
    xk = seeded_kv(41, 1, (1, 2, 200, 128), "f16", channel_scale=True)
    xv = seeded_kv(42, 1, (1, 2, 200, 128), "f16")
    kc = gear.Cache(p, 1, 2, 200, 2, TORCH_DT["f16"])
    vc = gear.Cache(p, 1, 2, 200, 2, TORCH_DT["f16"])
    gear.encode_batch([kc, vc], [to_dev(xk, "f16"), to_dev(xv, "f16")])
    q = seeded_kv(43, 1, (1, 2, 128), "f16")
    out = gear.decode_attn(kc, vc, to_dev(q, "f16"), 1.0 / math.sqrt(128), out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert gear.device_status() == 0
    op = oracle_params(p)
    for h in range(2):
        Kh = oracle.reconstruct_unit(oracle.encode_unit(xk[0, h], op), op)
        Vh = oracle.reconstruct_unit(oracle.encode_unit(xv[0, h], op), op)
        ref = oracle.attention(q[0, h].astype(np.float64), Kh, Vh, 1.0 / math.sqrt(128))
        vmax = np.abs(Vh).max()
        assert np.abs(out[0, h].cpu().numpy() - ref).max() <= 1e-3 * vmax
