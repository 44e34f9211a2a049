"""The seeded input generator: determinism, slices, distributions, storage rounding."""
import math

import numpy as np
import pytest
import scipy.stats
import torch

import synth
from synth import configs as C


def test_deterministic_and_slice_consistent():
    a = np.empty(10000, np.uint16)
    b = np.empty(10000, np.uint16)
    synth.fill_normal_host(a, 0, 42, 0.0, 0.3)
    synth.fill_normal_host(b, 0, 42, 0.0, 0.3)
    assert np.array_equal(a, b)
    part = np.empty(777, np.uint16)
    synth.fill_normal_host(part, 0, 42, 0.0, 0.3, offset=1234)
    assert np.array_equal(part, a[1234:1234 + 777])
    c = np.empty(10000, np.uint16)
    synth.fill_normal_host(c, 0, 43, 0.0, 0.3)
    assert not np.array_equal(a, c)


def test_normal_distribution():
    z = synth.normal_f64(400000, 0, 5)
    assert abs(z.mean()) < 0.01 and abs(z.var() - 1.0) < 0.01
    assert scipy.stats.kstest(z, "norm").pvalue > 1e-3


def test_series_functions_accuracy():
    L = synth._host_lib()
    rng = np.random.RandomState(0)
    for x in rng.uniform(1e-12, 1.0, 2000):
        assert abs(L.synth_log_f64(x) - math.log(x)) <= 1e-15 * abs(math.log(x)) + 1e-16
    for x in rng.uniform(-2.4, 2.4, 2000):
        assert abs(L.synth_exp_f64(x) / math.exp(x) - 1) <= 1e-15


def test_log_uniform_scale():
    s = synth.log_uniform_f64(200000, 0, C.TID_X_SCALE)
    assert s.min() >= 0.1 * (1 - 1e-12) and s.max() <= 10 * (1 + 1e-12)
    assert scipy.stats.kstest(np.log10(s), "uniform", args=(-1, 2)).pvalue > 1e-3


def test_bf16_rounding_matches_torch_on_f32_values():
    rng = np.random.RandomState(1)
    vals = (rng.randn(5000) * np.exp(rng.uniform(-8, 8, 5000))).astype(np.float32)
    ref = torch.tensor(vals).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    got = np.array([synth.f64_to_bf16_bits_scalar(float(v)) for v in vals], dtype=np.uint16)
    assert np.array_equal(got, ref)


def test_bf16_rounding_ties_to_even():
    # 1 + 2^-8 is halfway between bf16 1.0 and 1.0078125: ties go to the even mantissa (1.0)
    assert synth.f64_to_bf16_bits_scalar(1.0 + 2.0 ** -8) == 0x3F80
    # 1 + 3 * 2^-8 is halfway between 1.0078125 (odd) and 1.015625 (even)
    assert synth.f64_to_bf16_bits_scalar(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above the tie rounds up
    assert synth.f64_to_bf16_bits_scalar(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81


def test_layer_recipe_shapes_and_scales():
    cfg = C.CONFIGS["c2_bf16"]
    w = C.make_layer_host(cfg, 0)
    dims = C.mlp_dims(cfg)
    assert w["Y"].shape == (64, 16) and w["W_L"].shape == (32, 64)
    for j in range(len(dims) - 1):
        assert w["W%d" % j].shape == (dims[j + 1], dims[j])
        std = C.to_f64(w["W%d" % j]).std()
        assert abs(std * math.sqrt(dims[j]) - 1.0) < 0.02
    g = w["fmb_gamma"].astype(np.float64)
    assert abs(g.mean() - 1.0) < 0.005 and abs(g.std() - 0.02) < 0.003


def test_flops_per_example_matches_workload_labels():
    assert abs(C.flops_per_example(C.CONFIGS["c4_bf16"]) / 1e9 - 24.13) < 0.01
    assert abs(C.flops_per_example(C.CONFIGS["c3_bf16"]) / 1e9 - 1.137) < 0.001


def test_x_logscaled_rows_share_feature_scale():
    cfg = C.CONFIGS["c5_bf16"]
    X = C.to_f64(C.make_x_host(cfg, [0, 5]))
    s = synth.log_uniform_f64(cfg["n"], 0, C.TID_X_SCALE)
    z = synth.normal_f64(cfg["n"] * cfg["d"], 0, C.TID_X, offset=5 * cfg["n"] * cfg["d"]).reshape(cfg["n"], cfg["d"])
    ref = (s[:, None] * z)
    assert np.allclose(X[1], ref, rtol=2 ** -8, atol=0)


@pytest.mark.gpu
def test_device_fill_bit_identical_to_host(cuda_device):
    t = torch.empty(300001, dtype=torch.bfloat16, device=cuda_device)
    synth.fill_normal_dev(t, 0, 77, 0.0, 0.05, offset=99)
    h = np.empty(300001, np.uint16)
    synth.fill_normal_host(h, 0, 77, 0.0, 0.05, offset=99)
    assert np.array_equal(t.view(torch.int16).cpu().numpy().astype(np.uint16), h)
    f = torch.empty(50001, dtype=torch.float32, device=cuda_device)
    synth.fill_normal_dev(f, 3, 9, 1.0, 0.02)
    hf = np.empty(50001, np.float32)
    synth.fill_normal_host(hf, 3, 9, 1.0, 0.02)
    assert np.array_equal(f.cpu().numpy().view(np.uint32), hf.view(np.uint32))
    cfg = C.CONFIGS["c5_bf16"]
    xd = C.make_x_dev(cfg, 3, device=cuda_device, first_example=7)
    xh = C.make_x_host(cfg, [7, 8, 9])
    assert np.array_equal(xd.view(torch.int16).cpu().numpy().astype(np.uint16), xh)
