"""Whole-stack parity: the C-ABI forward of each workload, run on its full batch on
the GPU, against the fp64 oracle on sampled examples (per-example independence makes
the sample exact), plus batch-split and host-buffer consistency.

Tolerance (max over sampled outputs of |gpu - ref| / (1 + |ref|)): 1e-4 for the fp32
workload, 2e-2 for the bf16-in / fp32-accumulate workloads.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, max_scaled_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _sample(batch, count, seed=0):
    rng = np.random.RandomState(seed)
    fixed = [0, 1, batch // 2, batch - 1]
    rest = rng.choice(np.arange(2, batch - 1), size=max(0, count - len(fixed)), replace=False).tolist()
    return sorted(set(fixed + rest))[:count] if count < batch else list(range(batch))


class DevStack:
    def __init__(self, name, max_batch=None, operand_dtype=None):
        self.cfg = C.CONFIGS[name]
        self.layers = [C.make_layer_dev(self.cfg, l) for l in range(self.cfg["layers"])]
        self.h = wk.wk_stack_create(self.cfg, self.layers, max_batch=max_batch or self.cfg["batch"],
                                    operand_dtype=operand_dtype)

    def run(self, X):
        out = torch.empty_like(X)
        wk.wk_stack_forward(self.h, X, out)
        torch.cuda.synchronize()
        assert wk.wk_stack_sync_status(self.h) == wk.WK_OK
        return out

    def close(self):
        wk.wk_stack_destroy(self.h)
        self.layers = None


def _oracle(cfg, examples):
    X = C.to_f64(C.make_x_host(cfg, examples))
    return oracle.stack_forward(cfg, lambda l: C.make_layer_host(cfg, l), X)


def _parity(name, n_sample, operand_dtype=None):
    cfg = C.CONFIGS[name]
    st = DevStack(name, operand_dtype=operand_dtype)
    try:
        X = C.make_x_dev(cfg, cfg["batch"])
        out = st.run(X)
        ex = _sample(cfg["batch"], n_sample)
        got = f64(out[ex])
        assert np.isfinite(got).all()
        ref = _oracle(cfg, ex)
        err = max_scaled_err(got, ref)
        print("%s (operands %s): max |gpu-ref|/(1+|ref|) = %.3g over %d examples"
              % (name, operand_dtype or "default", err, len(ex)))
        assert err <= TOL[cfg["dtype"]]
    finally:
        st.close()
        torch.cuda.empty_cache()


def test_weights_device_generator_matches_host():
    for name in ("c1_fp32", "c5_bf16"):
        cfg = C.CONFIGS[name]
        dev = C.make_layer_dev(cfg, 1 if cfg["layers"] > 1 else 0)
        host = C.make_layer_host(cfg, 1 if cfg["layers"] > 1 else 0)
        for k in ("Y", "W_L", "W0"):
            d = dev[k].cpu()
            d = d.view(torch.int16).numpy().view(np.uint16) if d.dtype == torch.bfloat16 else d.numpy()
            assert np.array_equal(d, host[k]), (name, k)


def test_parity_c1_fp32_all_examples():
    _parity("c1_fp32", 64)


def test_parity_c2_bf16():
    _parity("c2_bf16", 512)


def test_parity_c2_bf16_with_bf16_operands():
    _parity("c2_bf16", 512, operand_dtype="bf16")


def test_parity_c5_bf16_wide_narrow():
    _parity("c5_bf16", 16)


def test_parity_c3_bf16():
    _parity("c3_bf16", 16)


def test_batch_split_is_bitwise_and_host_path_matches():
    cfg = C.CONFIGS["c2_bf16"]
    st = DevStack("c2_bf16")
    try:
        X = C.make_x_dev(cfg, cfg["batch"])
        full = st.run(X)
        a = st.run(X[:1000].contiguous())
        b = st.run(X[1000:].contiguous())
        assert torch.equal(torch.cat([a, b]), full)
        perm = torch.randperm(cfg["batch"], device=X.device)
        assert torch.equal(st.run(X[perm].contiguous()), full[perm])
        xh = X.cpu().pin_memory()
        oh = torch.empty_like(xh).pin_memory()
        wk.wk_stack_forward_host(st.h, xh, oh)
        assert torch.equal(oh, full.cpu())
    finally:
        st.close()


def test_profiling_counts_launches():
    cfg = C.CONFIGS["c2_bf16"]
    st = DevStack("c2_bf16")
    try:
        X = C.make_x_dev(cfg, 512)
        wk.wk_stack_set_profiling(st.h, True)
        st.run(X)
        t = wk.wk_stack_kernel_times(st.h)
        m = len(cfg["hidden"]) + 1
        assert t["fm_ln"][1] == cfg["layers"] and t["mlp_gemm"][1] == cfg["layers"] * m
        # the residual + LayerNorm runs in its own kernel, or inside the last Linear and LCB epilogues
        assert t["lcb"][1] == cfg["layers"] and t["res_ln"][1] in (0, cfg["layers"])
        assert all(ms > 0 for ms, count in t.values() if count)
    finally:
        st.close()


def test_parity_c4_bf16_full_size():
    _parity("c4_bf16", 16)
