"""The seeded input generator gives identical values on its numpy (oracle) side
and its torch (device) side, so both sides of a parity test see the same data."""
import numpy as np
import torch

import workloads as wl


def test_normal_numpy_equals_torch():
    idx = np.concatenate([np.arange(5000), np.arange(2**32 - 100, 2**32 + 100), [2**40 + 7]]).astype(np.int64)
    a = wl.normal_np(1234, 3, idx)
    b = wl.normal_torch(1234, 3, torch.from_numpy(idx)).numpy()
    assert np.array_equal(a, b)
    assert abs(a[:5000].mean()) < 0.05 and abs(a[:5000].std() - 1) < 0.05
    assert np.abs(a).max() <= 3.47


def test_units_match_tensor_slices():
    for name in ["tiny", "llama7b_layer_encode", "llama3_8b_gqa"]:
        w = wl.WORKLOADS[name]
        n = 40
        for which in ["k", "v"]:
            t = wl.kv_tensor_torch(w, which, 0, "cpu", n=n)
            t32 = t.float().numpy()
            for b, h in [(0, 0), (w.B - 1, w.H - 1)]:
                u = wl.kv_unit_np(w, which, 0, b, h, n=n)
                assert np.array_equal(u, t32[b, h]), (name, which, b, h)
    w = wl.WORKLOADS["decode_b16_ctx8192"]
    assert np.array_equal(wl.rows_np(w, wl.S_Q, 0, 0, w.Hq),
                          wl.rows_torch(w, wl.S_Q, 0, 0, w.Hq, "cpu").float().numpy())


def test_tiny_spikes_and_channel_scale():
    w = wl.WORKLOADS["tiny"]
    sp = wl.spike_positions(w)
    assert sp.size == round(0.01 * 256 * 128) and np.unique(sp).size == sp.size
    sig = wl.channel_sigma(wl.WORKLOADS["llama7b_layer_encode"], 0)
    assert sig.min() >= 0.5 and sig.max() <= 8.0


def test_tiny_draws_true_normals():
    """The tiny codec workload asks for i.i.d. N(0,1) entries: its values come from
    numpy's seeded generator (unbounded tails), identical on both sides."""
    w = wl.WORKLOADS["tiny"]
    v = wl.kv_unit_np(w, "v", 0, 0, 0)
    assert v.shape == (256, 128) and abs(v.mean()) < 0.05 and abs(v.std() - 1) < 0.05
    assert np.abs(v).max() > 3.47    # beyond the bounded Irwin-Hall support
    k = wl.kv_unit_np(w, "k", 0, 0, 0)
    sp = wl.spike_positions(w)
    base = np.random.default_rng([w.seed, wl.S_K, 0, 0, 0]).standard_normal((256, 128), dtype=np.float32)
    assert np.array_equal(k.reshape(-1)[sp], base.reshape(-1)[sp] * np.float32(10.0))
    mask = np.ones(256 * 128, bool)
    mask[sp] = False
    assert np.array_equal(k.reshape(-1)[mask], base.reshape(-1)[mask])
    assert np.array_equal(wl.rows_np(w, wl.S_Q, 0, 0, 1), wl.rows_torch(w, wl.S_Q, 0, 0, 1, "cpu").numpy())
