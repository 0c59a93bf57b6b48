"""The seeded input generator: shapes, determinism and bf16 rounding."""

import numpy as np
import torch

from selective_state_space_silu_b200 import inputs as I


def test_bf16_rounding_matches_torch():
    r = np.random.default_rng(0)
    a = np.concatenate([r.standard_normal(100000).astype(np.float32) * 10 ** r.uniform(-30, 30, 100000).astype(np.float32),
                        np.array([0.0, -0.0, np.inf, -np.inf, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8,
                                  3.3895314e38], dtype=np.float32)]).astype(np.float32)
    ours = I.f32_to_bf16_bits(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = I.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(a).to(torch.bfloat16).float().numpy())


def test_shapes_and_determinism():
    w = I.WORKLOADS["tiny"]
    a = I.make_inputs(w)
    b = I.make_inputs(w)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["xp"].shape == (2, 16, 128) and a["B"].shape == (2, 16, 16)
    assert a["A_log"].shape == (128, 16) and a["conv_w"].shape == (128, 4)
    np.testing.assert_allclose(a["A_log"][5], np.log(np.arange(1, 17)), rtol=1e-7)
    dec = I.make_inputs(I.WORKLOADS["decode"].with_(batch=4, d_inner=64))
    assert dec["h"].shape == (4, 64, 16) and dec["conv_state"].shape == (4, 64, 3)
    assert dec["xp"].dtype == np.uint16


def test_distributions():
    w = I.WORKLOADS["stress"]
    a = I.make_inputs(w)
    assert abs(a["xp"].std() - 1.0) < 0.01 and abs(a["dt_raw"].std() - 0.5) < 0.01
    dt0 = np.logaddexp(0.0, a["dt_bias"].astype(np.float64))   # softplus(dt_bias) = dt0
    assert dt0.min() >= 1e-3 * (1 - 1e-5) and dt0.max() <= 1e-1 * (1 + 1e-5)
    assert np.all(np.abs(a["conv_w"]) <= 0.5) and np.all(a["D"] == 1.0)


def test_ssd_inputs_shapes_determinism_distributions():
    w = I.SsdWorkload("t", 3, 50, 6, 64, 128, 2, 77, gate=True, state=True)
    a = I.make_ssd_inputs(w)
    b = I.make_ssd_inputs(w)
    for k in a:
        np.testing.assert_array_equal(a[k], b[k])
    assert a["x"].shape == (3, 50, 6, 64) and a["z"].shape == (3, 50, 6, 64)
    assert a["dt_raw"].shape == (3, 50, 6) and a["B"].shape == (3, 50, 2, 128)
    assert a["A_log"].shape == (6,) and a["h_in"].shape == (3, 6, 64, 128)
    assert a["x"].dtype == np.uint16 and a["h_in"].dtype == np.float32
    A = np.exp(a["A_log"].astype(np.float64))
    assert (A >= 1.0 - 1e-6).all() and (A <= 16.0 + 1e-5).all()
    dt0 = np.logaddexp(0.0, a["dt_bias"].astype(np.float64))
    assert dt0.min() >= 1e-3 * (1 - 1e-5) and dt0.max() <= 1e-1 * (1 + 1e-5)
    big = I.make_ssd_inputs(I.SsdWorkload("u", 4, 512, 8, 64, 64, 1, 78))
    x = I.bf16_bits_to_f32(big["x"])
    assert abs(x.std() - 1.0) < 0.01 and big["z"] is None and big["h_in"] is None
    assert abs(I.bf16_bits_to_f32(big["dt_raw"]).std() - 0.5) < 0.02
