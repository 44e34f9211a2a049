"""Each step of a Wukong layer alone (stand-alone C-ABI entry points) against the
fp64 oracle's matching step, on the same generator bits, at sizes that span several
tiles and ragged tails."""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from tests.gpu_util import f64, host_normal, max_scaled_err, oracle_weight, to_dev, torch_dtype

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _status_ok():
    torch.cuda.synchronize()
    assert wk.wk_device_status() == wk.WK_OK


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("M,K,N,relu,bias", [
    (128, 64, 256, False, False),      # one tile, one k-block
    (333, 264, 520, True, True),       # ragged M, K (not a multiple of 64) and N
    (1000, 1024, 768, True, True),     # several tiles per CTA
    (64, 4096, 256, False, True),      # long K, M below one tile
])
def test_mlp_linear_tcgen05(M, K, N, relu, bias, dt):
    A = host_normal((M, K), 1, dtype=dt)
    W = host_normal((N, K), 2, std=1.0 / np.sqrt(K), dtype=dt)
    b = host_normal((N,), 3, std=0.5, dtype="f32") if bias else None
    C = torch.full((M, N), float("nan"), dtype=torch_dtype(dt), device="cuda")
    wk.wk_mlp_linear(to_dev(A), to_dev(W), to_dev(b) if bias else None, C, M, K, N, N, relu, dt)
    _status_ok()
    ref = oracle.linear(f64(A), oracle_weight(W), b, relu=relu)
    got = f64(C)
    scale = np.sqrt(np.mean(ref ** 2))
    rel = 2.0 ** -8 if dt == "bf16" else 2.0 ** -10
    assert np.all(np.abs(got - ref) <= rel * np.abs(ref) + 2e-3 * scale)


def test_mlp_linear_row_stride_into_wider_buffer():
    M, K, N, ldc = 200, 128, 256, 640
    A = host_normal((M, K), 4)
    W = host_normal((N, K), 5, std=1.0 / np.sqrt(K))
    C = torch.zeros((M, ldc), dtype=torch.bfloat16, device="cuda")
    wk.wk_mlp_linear(to_dev(A), to_dev(W), None, C, M, K, N, ldc, False, "bf16")
    _status_ok()
    ref = oracle.linear(f64(A), W)
    got = f64(C)
    assert np.all(got[:, N:] == 0.0)
    assert np.all(np.abs(got[:, :N] - ref) <= 2.0 ** -8 * np.abs(ref) + 2e-3 * np.sqrt(np.mean(ref ** 2)))


def test_mlp_linear_f32_simt():
    M, K, N = 70, 64, 136
    A = host_normal((M, K), 6, dtype="f32")
    W = host_normal((N, K), 7, std=0.125, dtype="f32")
    b = host_normal((N,), 8, dtype="f32")
    C = torch.empty((M, N), dtype=torch.float32, device="cuda")
    wk.wk_mlp_linear(to_dev(A), to_dev(W), to_dev(b), C, M, K, N, N, True, "f32")
    _status_ok()
    ref = oracle.linear(f64(A), W, b, relu=True)
    assert max_scaled_err(f64(C), ref) <= 1e-5


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("batch,n,d,n_f,n_l", [
    (5, 512, 160, 256, 256),   # one example per tile (E = 1), two W_L tiles
    (13, 720, 32, 360, 360),   # E = 8 with a ragged group, K tail (720 = 11*64 + 16), M tail (360)
    (7, 64, 128, 32, 32),      # E = 2, ragged group
    (9, 128, 64, 64, 64),      # E = 4 examples x 2 column chunks per copy, ragged group
    (11, 96, 96, 48, 48),      # E = 2 examples x 3 column chunks per copy, K and M tails
    (301, 512, 160, 256, 256),  # resident W_L: several example groups per CTA, the X ring wraps
    (1000, 256, 160, 128, 128),  # resident W_L, one m tile for every CTA
    (97, 200, 160, 100, 100),  # resident W_L with a K tail (200 = 3*64 + 8) and an M tail (100 rows)
])
def test_lcb_tcgen05(batch, n, d, n_f, n_l, dt):
    WL = host_normal((n_l, n), 9, std=1.0 / np.sqrt(n), dtype=dt)
    X = host_normal((batch, n, d), 10, dtype=dt)
    cat = torch.full((batch, n_f + n_l, d), 7.0, dtype=torch_dtype(dt), device="cuda")
    wk.wk_lcb(to_dev(WL), to_dev(X), cat, batch, n, d, n_f, n_l, dt)
    _status_ok()
    got = f64(cat)
    assert np.all(got[:, :n_f] == 7.0)  # FMB rows untouched
    for b in range(batch):
        ref = oracle.lcb(f64(WL), f64(X[b]))
        err = np.abs(got[b, n_f:] - ref)
        assert np.all(err <= 2.0 ** -8 * np.abs(ref) + 2e-3 * np.sqrt(np.mean(ref ** 2))), b


def test_lcb_f32_simt():
    batch, n, d, n_f, n_l = 6, 16, 16, 8, 8
    WL = host_normal((n_l, n), 12, std=0.25, dtype="f32")
    X = host_normal((batch, n, d), 13, dtype="f32")
    cat = torch.zeros((batch, n, d), dtype=torch.float32, device="cuda")
    wk.wk_lcb(to_dev(WL), to_dev(X), cat, batch, n, d, n_f, n_l, "f32")
    _status_ok()
    got = f64(cat)
    for b in range(batch):
        assert max_scaled_err(got[b, n_f:], oracle.lcb(f64(WL), f64(X[b]))) <= 1e-5


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("batch,n,d,k", [
    (300, 512, 160, 64),   # more examples than SMs: persistent CTAs take several
    (150, 256, 160, 32),
    (200, 64, 128, 16),
    (170, 720, 32, 24),    # tail chunk of 80 rows
])
def test_fm_ln_mma(batch, n, d, k, dt):
    X = host_normal((batch, n, d), 14, dtype=dt)
    Y = host_normal((n, k), 15, std=1.0 / np.sqrt(n), dtype=dt)
    g = host_normal((n * k,), 16, mean=1.0, std=0.1, dtype="f32")
    be = host_normal((n * k,), 17, std=0.1, dtype="f32")
    A0 = torch.full((batch, n * k), float("nan"), dtype=torch_dtype(dt), device="cuda")
    wk.wk_fm_ln(to_dev(X), to_dev(Y), to_dev(g), to_dev(be), A0, batch, n, d, k, dt)
    _status_ok()
    got = f64(A0)
    for b in list(range(0, batch, max(1, batch // 12))) + [batch - 1]:
        F = oracle.fm(f64(X[b]), f64(Y))
        ref = oracle.layernorm(F.reshape(-1), f64(g), f64(be))
        assert max_scaled_err(got[b], ref) <= (1.5e-2 if dt == "bf16" else 4e-3), b


def test_fm_ln_f32_simt():
    batch, n, d, k = 9, 16, 16, 4
    X = host_normal((batch, n, d), 18, dtype="f32")
    Y = host_normal((n, k), 19, std=0.25, dtype="f32")
    g = host_normal((n * k,), 20, mean=1.0, std=0.1, dtype="f32")
    be = host_normal((n * k,), 21, std=0.1, dtype="f32")
    A0 = torch.empty((batch, n * k), dtype=torch.float32, device="cuda")
    wk.wk_fm_ln(to_dev(X), to_dev(Y), to_dev(g), to_dev(be), A0, batch, n, d, k, "f32")
    _status_ok()
    got = f64(A0)
    for b in range(batch):
        ref = oracle.layernorm(oracle.fm(f64(X[b]), f64(Y)).reshape(-1), f64(g), f64(be))
        assert max_scaled_err(got[b], ref) <= 1e-4


# Row counts: ragged against every stage size of the bulk-copy ring (R = 32..512 rows)
# and, for the largest, several laps of the ring on every SM.
@pytest.mark.parametrize("rows,d,dt", [(1003, 160, "bf16"), (4097, 32, "bf16"), (515, 128, "bf16"),
                                       (333, 16, "f32"), (100, 256, "bf16"), (1003, 160, "f16"),
                                       (40001, 160, "f16"), (2999, 192, "f16"), (777, 64, "bf16"),
                                       (1501, 16, "f16"), (5, 160, "f16")])
def test_res_ln(rows, d, dt):
    cat = host_normal((rows, d), 22, dtype=dt)
    X = host_normal((rows, d), 23, dtype=dt)
    g = host_normal((d,), 24, mean=1.0, std=0.2, dtype="f32")
    be = host_normal((d,), 25, std=0.2, dtype="f32")
    out = torch.empty((rows, d), dtype=torch_dtype(dt), device="cuda")
    wk.wk_res_ln(to_dev(cat), to_dev(X), to_dev(g), to_dev(be), out, rows, d, dt)
    _status_ok()
    got = f64(out)
    y = f64(cat) + f64(X)
    tol = {"bf16": 1e-2, "f16": 2e-3, "f32": 1e-5}[dt]
    for r in range(rows):
        assert max_scaled_err(got[r], oracle.layernorm(y[r], f64(g), f64(be))) <= tol, r


@pytest.mark.parametrize("batch,n,d,k", [(160, 512, 160, 64), (170, 720, 32, 24), (150, 256, 160, 32), (200, 64, 128, 16)])
def test_fm_ln_without_affine(batch, n, d, k):
    """NULL gamma/beta: A0 holds the normalised FM values (how a stack calls it)."""
    X = host_normal((batch, n, d), 26, dtype="f16")
    Y = host_normal((n, k), 27, std=1.0 / np.sqrt(n), dtype="f16")
    A0 = torch.full((batch, n * k), float("nan"), dtype=torch.float16, device="cuda")
    wk.wk_fm_ln(to_dev(X), to_dev(Y), None, None, A0, batch, n, d, k, "f16")
    _status_ok()
    got = f64(A0)
    for b in (0, batch // 2, batch - 1):
        ref = oracle.layernorm(oracle.fm(f64(X[b]), f64(Y)).reshape(-1))
        assert max_scaled_err(got[b], ref) <= 4e-3, b
