"""The seeded input generators on CPU: rows regenerate independently, bf16
rounding is round-to-nearest-even, and the draws have the distributions the
workloads state. No GPU."""
import numpy as np
import torch

from wkv_recurrence_b200 import inputs as I


def test_rows_regenerate_independently():
    wl = I.WORKLOADS["layer"]
    k, v = I.draw_kv_rows(wl, range(wl.B), T=1100)  # three 512-token blocks, the last partial
    ks, vs = I.draw_kv_rows(wl, [5, 2], T=1100)
    assert np.array_equal(ks, k[[5, 2]]) and np.array_equal(vs, v[[5, 2]])
    k2, _ = I.draw_kv_rows(wl, range(wl.B), T=1100)
    assert np.array_equal(k, k2)  # deterministic
    k3, _ = I.draw_kv_rows(wl, range(wl.B), seed=1, T=1100)
    assert not np.array_equal(k, k3)  # the seed matters
    dk, dv = I.draw_decode_token(I.WORKLOADS["decode"], 7, rows=range(16))
    sk, sv = I.draw_decode_token(I.WORKLOADS["decode"], 7, rows=[9, 3])
    assert np.array_equal(sk, dk[[9, 3]]) and np.array_equal(sv, dv[[9, 3]])
    n, d, m = I.draw_state(I.WORKLOADS["mixed"], rows=range(4))
    n2, d2, m2 = I.draw_state(I.WORKLOADS["mixed"], rows=[3])
    assert np.array_equal(n2, n[[3]]) and np.array_equal(d2, d[[3]]) and np.array_equal(m2, m[[3]])


def test_bf16_rounding_is_nearest_even():
    one = 1.0
    cases = {
        one: 0x3F80,
        one + 2.0 ** -8: 0x3F80,                # halfway: ties to the even code
        one + 3 * 2.0 ** -8: 0x3F82,            # halfway: ties to the even code (up)
        one + 2.0 ** -8 + 2.0 ** -20: 0x3F81,   # just above halfway
        -2.0: 0xC000,
        0.0: 0x0000,
    }
    for x, code in cases.items():
        assert int(I.f32_to_bf16_bits(np.array([x], np.float32))[0]) == code, x
    # against torch's own fp32 -> bf16 conversion (round to nearest even)
    g = np.random.default_rng(5)
    x = (g.standard_normal(100_000) * np.exp(g.uniform(-20, 20, 100_000))).astype(np.float32)
    ours = I.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(ours, ref)
    back = I.bf16_bits_to_f32(ours)
    assert np.array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())
    assert np.all(np.abs(back - x) <= np.abs(x) * 2.0 ** -8)


def test_parameter_distributions():
    w = I.draw_w(I.WORKLOADS["layer"])
    assert w.dtype == np.float32 and w.min() >= 1e-3 and w.max() <= 8.0
    lw = np.log(w.astype(np.float64))
    assert abs(np.median(lw) - (-1.0)) < 0.15  # log-normal around -1, clipped
    wl = I.draw_w(I.WORKLOADS["long"]).astype(np.float64)
    assert wl.min() >= 1e-4 * (1 - 1e-6) and wl.max() <= 4.0 * (1 + 1e-6)
    lo, hi = np.log(1e-4), np.log(4.0)
    assert abs(np.mean(np.log(wl)) - (lo + hi) / 2) < 0.4  # log-uniform: mean of the log at the midpoint
    u = I.draw_u(I.WORKLOADS["mixed"]).astype(np.float64)
    assert abs(u.mean()) < 0.03 and abs(u.std() - 0.5) < 0.03  # N(0, 0.5): sigma 0.5


def test_key_distributions():
    k, v = I.draw_kv_rows(I.WORKLOADS["long"], [0], T=2048)
    spikes = np.abs(k) >= 20.0
    frac = spikes.mean()
    assert 0.009 < frac < 0.011  # 1% of keys
    assert np.abs(k[spikes]).max() <= 60.0
    assert abs(v.mean()) < 0.01 and abs(v.std() - 1.0) < 0.01
    kb, _ = I.draw_kv_rows(I.WORKLOADS["mixed"], [0], T=512)
    assert kb.dtype == np.uint16
    kf = I.bf16_bits_to_f32(kb).astype(np.float64)
    # 2 x Student-t(3): median |k| = 2 x 0.7649 (the t3 quartile)
    assert abs(np.median(np.abs(kf)) - 2 * 0.7649) < 0.02
    assert np.abs(kf).max() > 20.0  # heavy tails


def test_random_state_is_valid():
    n, d, m = I.draw_state(I.WORKLOADS["mixed"], rows=range(2))
    assert d.min() >= 1.0 and d.max() <= 16.0
    assert np.all(np.abs(n) <= d * 4.0)  # num = den * N(0, 0.5)
    assert I.draw_state(I.WORKLOADS["layer"]) is None  # the zero state
