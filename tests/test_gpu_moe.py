"""Wukong mixture of experts on the GPU (Kunlun page, section 2.3, "Wukong Mixture of
Experts"; reading: MoE(X) = sum_e softmax(W_g vec(X) + b_g)_e WukongLayer_e(X)) against
the fp64 oracle: the gate kernel and the combine kernel alone, then whole MoE stacks
through the C ABI on sampled examples, plus batch-split consistency.

Tolerances: the gate is fp32 arithmetic on 16-bit inputs (absolute 1e-4 on weights
in [0, 1]); the combine output is one 16-bit rounding of an fp32 mixture (relative
2^-8 bf16 / 2^-10 fp16 plus a small absolute term); whole stacks use the stack
tolerance of the bf16 workloads, max |gpu - ref| / (1 + |ref|) <= 2e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, host_normal, max_scaled_err, to_dev, torch_dtype

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
@pytest.mark.parametrize("batch,nd,E,bias", [(1, 8, 1, False), (333, 8192, 5, True), (64, 40960, 8, True),
                                             (7, 2048, 2, False)])
def test_gate_kernel(batch, nd, E, bias, dt):
    X = host_normal((batch, nd), 21, dtype=dt)
    W = host_normal((E, nd), 22, std=1.0 / np.sqrt(nd), dtype=dt)
    b = host_normal((E,), 23, dtype="f32") if bias else None
    g = torch.full((batch, E), float("nan"), dtype=torch.float32, device="cuda")
    wk.wk_moe_gate_softmax(to_dev(X), to_dev(W), to_dev(b) if bias else None, g, batch, nd, E, dt)
    _status_ok()
    ref = oracle.gate_softmax(W.astype(np.float32) if dt == "f16" else W, b, f64(X).reshape(batch, nd, 1))
    got = g.double().cpu().numpy()
    assert np.allclose(got.sum(axis=1), 1.0, atol=1e-5)
    assert np.max(np.abs(got - ref)) <= 1e-4


@pytest.mark.parametrize("dt", ["bf16", "f16"])
@pytest.mark.parametrize("batch,n,d,E", [(37, 64, 128, 3), (5, 512, 160, 4), (19, 720, 32, 2), (3, 16, 16, 8),
                                         (11, 256, 160, 1)])
def test_combine_kernel(batch, n, d, E, dt):
    cats = [host_normal((batch, n, d), 30 + e, dtype=dt) for e in range(E)]
    X = host_normal((batch, n, d), 40, dtype=dt)
    logits = host_normal((batch, E), 41, dtype="f32")
    gw = np.exp(logits - logits.max(axis=1, keepdims=True))
    gw = (gw / gw.sum(axis=1, keepdims=True)).astype(np.float32)
    gam = [host_normal((d,), 50 + e, mean=1.0, std=0.2, dtype="f32") for e in range(E)]
    bet = [host_normal((d,), 60 + e, std=0.2, dtype="f32") for e in range(E)]
    out = torch.full((batch, n, d), float("nan"), dtype=torch_dtype(dt), device="cuda")
    dcats = [to_dev(c) for c in cats]
    dg = [to_dev(t) for t in gam]
    db = [to_dev(t) for t in bet]
    wk.wk_moe_combine(dcats, to_dev(X), to_dev(gw), dg, db, out, batch, n, d, dt)
    _status_ok()
    x64 = f64(X)
    ref = np.zeros((batch, n, d))
    for e in range(E):
        y = f64(cats[e]) + x64
        mu = y.mean(axis=2, keepdims=True)
        var = ((y - mu) ** 2).mean(axis=2, keepdims=True)
        ln = (y - mu) / np.sqrt(var + 1e-5) * gam[e].astype(np.float64) + bet[e].astype(np.float64)
        ref += gw[:, e].astype(np.float64)[:, None, None] * ln
    # spot-check the numpy LayerNorm above against the oracle's on a few rows
    for (b, i) in [(0, 0), (batch - 1, n - 1)]:
        y = f64(cats[0])[b, i] + x64[b, i]
        assert np.allclose(oracle.layernorm(y, gam[0], bet[0]),
                           (y - y.mean()) / np.sqrt(((y - y.mean()) ** 2).mean() + 1e-5) * gam[0] + bet[0],
                           rtol=0, atol=1e-12)
    got = f64(out)
    rel = 2.0 ** -8 if dt == "bf16" else 2.0 ** -10
    assert np.all(np.abs(got - ref) <= rel * np.abs(ref) + 2e-4 * (1 + np.abs(ref)) + 1e-3)


class DevMoe:
    def __init__(self, name, max_batch=None, operand_dtype=None):
        self.cfg = C.MOE_CONFIGS[name]
        cfg = self.cfg
        self.experts = [[C.make_expert_dev(cfg, l, e) for e in range(cfg["experts"])] for l in range(cfg["layers"])]
        self.gates = [C.make_gate_dev(cfg, l) for l in range(cfg["layers"])]
        self.h = wk.wk_moe_create(cfg, self.experts, self.gates, max_batch=max_batch or cfg["batch"],
                                  operand_dtype=operand_dtype)

    def run(self, X):
        out = torch.empty_like(X)
        wk.wk_moe_forward(self.h, X, out)
        torch.cuda.synchronize()
        assert wk.wk_moe_sync_status(self.h) == wk.WK_OK
        return out

    def close(self):
        wk.wk_moe_destroy(self.h)
        self.experts = self.gates = None


def _moe_oracle(cfg, examples):
    X = C.to_f64(C.make_x_host(cfg, examples))
    return oracle.moe_forward(cfg, lambda l, e: C.make_expert_host(cfg, l, e), lambda l: C.make_gate_host(cfg, l), X)


def _sample(batch, count, seed=0):
    rng = np.random.RandomState(seed)
    fixed = [0, 1, batch // 2, batch - 1]
    rest = rng.choice(np.arange(2, batch - 1), size=max(0, count - len(fixed)), replace=False).tolist()
    return sorted(set(fixed + rest))[:count]


@pytest.mark.parametrize("name,n_sample,operand_dtype", [("moe3_c2", 64, None), ("moe3_c2", 64, "bf16"),
                                                         ("moe4_c3", 16, None)])
def test_moe_stack_parity(name, n_sample, operand_dtype):
    st = DevMoe(name, operand_dtype=operand_dtype)
    try:
        cfg = st.cfg
        X = C.make_x_dev(cfg, cfg["batch"])
        out = st.run(X)
        ex = _sample(cfg["batch"], n_sample)
        got = f64(out[ex])
        assert np.isfinite(got).all()
        ref = _moe_oracle(cfg, ex)
        err = max_scaled_err(got, ref)
        print("%s (operands %s): max |gpu-ref|/(1+|ref|) = %.3g over %d examples"
              % (name, operand_dtype or "default", err, len(ex)))
        assert err <= 2e-2
    finally:
        st.close()
        torch.cuda.empty_cache()


def test_moe_batch_split_is_bitwise_and_profiling_counts():
    st = DevMoe("moe3_c2")
    try:
        cfg = st.cfg
        X = C.make_x_dev(cfg, cfg["batch"])
        wk.wk_moe_set_profiling(st.h, True)
        full = st.run(X)
        t = wk.wk_moe_kernel_times(st.h)
        L, E, m = cfg["layers"], cfg["experts"], len(cfg["hidden"]) + 1
        assert t["moe_gate"][1] == L and t["moe_combine"][1] == L
        assert t["fm_ln"][1] == L * E and t["lcb"][1] == L * E and t["mlp_gemm"][1] == L * E * m
        assert t["res_ln"][1] == 0
        wk.wk_moe_set_profiling(st.h, False)
        a = st.run(X[:700].contiguous())
        b = st.run(X[700:].contiguous())
        assert torch.equal(torch.cat([a, b]), full)
    finally:
        st.close()
