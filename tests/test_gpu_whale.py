"""WHALE attention-based fusion on the GPU against the fp64 oracle (WHALE pages, section
2.1 item 3 and section 2.2). Reading: one head, K = V = H_s, A = softmax_rows(H_w H_s^T /
sqrt(d)) H_s; Z = [H_w | A] W_F^T + b_F; H_f = Z + (SiLU(U) * U) W_down^T, U = LN(Z) W_up^T.

The attention kernel alone on ragged and degenerate shapes (one key, one query, L one
past a block, peaked softmax weights that make the kernel raise its running max in the
middle of a row), the fusion + FFN kernel alone, and the two WHALE workloads through the
handle on sampled examples, plus batch-split consistency.

Tolerance: max |gpu - ref| / (1 + |ref|) <= 2e-2, the bound of the bf16-in /
fp32-accumulate workloads; the kernels round the softmax weights and the gated
activations to the 16-bit operand type.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, host_normal, max_scaled_err, oracle_weight, to_dev, torch_dtype

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _status_ok():
    torch.cuda.synchronize()
    assert wk.wk_device_status() == wk.WK_OK


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("batch,n,L,d,qstd", [
    (3, 64, 2048, 128, 1.0),    # queries of the 2-layer shape over 2048 positions
    (2, 512, 4096, 160, 1.0),   # queries of the 8-layer shape over 4096 positions
    (2, 200, 1000, 160, 6.0),   # ragged n and L; peaked weights raise the running max mid-row
    (5, 16, 130, 64, 3.0),      # 16 queries; L one key past a block
    (4, 130, 1, 32, 1.0),       # one key: A is that key
    (1, 1, 300, 128, 10.0),     # one query, nearly one-hot weights
    (3, 300, 640, 32, 4.0),
])
def test_attention_kernel(batch, n, L, d, qstd, dt):
    Hw = host_normal((batch, n, d), 101, std=qstd, dtype=dt)
    Hs = host_normal((batch, L, d), 102, dtype=dt)
    A = torch.full((batch, n, d), float("nan"), dtype=torch_dtype(dt), device="cuda")
    wk.wk_whale_attention(to_dev(Hw), to_dev(Hs), A, batch, n, L, d, dt)
    _status_ok()
    got = f64(A)
    hw, hs = f64(Hw), f64(Hs)
    ref = np.stack([oracle.attention_shared_kv(hw[b], hs[b]) for b in range(batch)])
    assert np.isfinite(got).all()
    err = max_scaled_err(got, ref)
    print("attention", batch, n, L, d, qstd, dt, "max scaled err %.2e" % err)
    assert err <= TOL
    if L == 1:  # every weight is exactly 1
        assert np.array_equal(got, np.broadcast_to(hs[:, :1, :], got.shape))


def _ffn_weights(d, h, bias, dt):
    return {"W_F": host_normal((d, 2 * d), 113, std=1.0 / np.sqrt(2 * d), dtype=dt),
            "b_F": host_normal((d,), 114, std=0.1, dtype="f32") if bias else None,
            "ln_gamma": host_normal((d,), 115, mean=1.0, std=0.1, dtype="f32"),
            "ln_beta": host_normal((d,), 116, std=0.1, dtype="f32"),
            "W_up": host_normal((h, d), 117, std=1.0 / np.sqrt(d), dtype=dt),
            "W_down": host_normal((d, h), 118, std=1.0 / np.sqrt(h), dtype=dt)}


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("rows,d,h,bias", [(300, 160, 640, True), (1000, 128, 512, True), (129, 64, 128, False),
                                           (77, 32, 64, True), (128, 160, 64, False), (5, 128, 192, True)])
def test_fusion_ffn_kernel(rows, d, h, bias, dt):
    Hw = host_normal((rows, d), 111, dtype=dt)
    A = host_normal((rows, d), 112, std=0.5, dtype=dt)
    w = _ffn_weights(d, h, bias, dt)
    dw = {k: (to_dev(v) if v is not None else None) for k, v in w.items()}
    Hf = torch.full((rows, d), float("nan"), dtype=torch_dtype(dt), device="cuda")
    wk.wk_whale_fusion_ffn(to_dev(Hw), to_dev(A), dw, Hf, rows, d, h, dt)
    _status_ok()
    ow = {k: (oracle_weight(v) if v is not None else None) for k, v in w.items()}
    ref = oracle.fusion_ffn(f64(Hw), f64(A), ow)
    got = f64(Hf)
    assert np.isfinite(got).all()
    err = max_scaled_err(got, ref)
    print("fusion+ffn", rows, d, h, bias, dt, "max scaled err %.2e" % err)
    assert err <= TOL


@pytest.mark.parametrize("name,sample", [("whale_c2", [0, 1, 511, 1023]), ("whale_c4", [0, 3, 128, 255])])
def test_whale_forward_workloads(name, sample):
    cfg = C.WHALE_CONFIGS[name]
    B = cfg["batch"]
    dw = C.make_whale_dev(cfg)
    h = wk.wk_whale_create(cfg, dw)
    Hw, Hs = C.make_whale_inputs_dev(cfg, B)
    Hf = torch.full_like(Hw, float("nan"))
    wk.wk_whale_forward(h, Hw, Hs, Hf)
    assert wk.wk_whale_sync_status(h) == wk.WK_OK
    hw, hs = C.make_whale_inputs_host(cfg, sample)
    assert np.array_equal(f64(Hw[sample]), f64(hw))  # the device generator gives the host's values
    hostw = C.make_whale_host(cfg)
    got = f64(Hf[sample])
    err = 0.0
    for r in range(len(sample)):
        ref = oracle.whale_fusion(f64(hw[r]), f64(hs[r]), hostw)
        err = max(err, max_scaled_err(got[r], ref))
    print(name, "max scaled err %.2e over examples %s" % (err, sample))
    assert err <= TOL
    # the first half of the batch alone gives the same rows, bit for bit
    half = B // 2
    Hf2 = torch.full_like(Hw, float("nan"))
    wk.wk_whale_forward(h, Hw[:half], Hs[:half], Hf2[:half])
    assert wk.wk_whale_sync_status(h) == wk.WK_OK
    assert torch.equal(Hf2[:half], Hf[:half])
    wk.wk_whale_destroy(h)


@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_attention_planted_key(dt):
    """A key in the last block scores far above every earlier key for query 0 (about 10 sqrt(d)
    per unit of |q|^2 / d): the kernel's weights from the running max are discarded and
    recomputed, and query 0 attends to that key alone."""
    batch, n, L, d = 3, 130, 700, 128
    Hw = host_normal((batch, n, d), 121, dtype="f32")
    Hs = host_normal((batch, L, d), 122, dtype="f32")
    Hs[:, L - 5, :] = 10.0 * Hw[:, 0, :]
    cast = (lambda a: a.astype(np.float16)) if dt == "f16" else (lambda a: _to_bf16_bits(a))
    Hw16, Hs16 = cast(Hw), cast(Hs)
    A = torch.full((batch, n, d), float("nan"), dtype=torch_dtype(dt), device="cuda")
    wk.wk_whale_attention(to_dev(Hw16), to_dev(Hs16), A, batch, n, L, d, dt)
    _status_ok()
    got = f64(A)
    hw, hs = f64(Hw16), f64(Hs16)
    ref = np.stack([oracle.attention_shared_kv(hw[b], hs[b]) for b in range(batch)])
    assert np.isfinite(got).all()
    assert np.allclose(ref[:, 0, :], hs[:, L - 5, :], rtol=0, atol=1e-9)  # the oracle: one-hot on that key
    err = max_scaled_err(got, ref)
    print("planted key", dt, "max scaled err %.2e" % err)
    assert err <= TOL


def _to_bf16_bits(a):
    """float32 -> bf16 bit patterns, round to nearest even."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)
