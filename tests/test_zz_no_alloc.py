"""The no-allocation one-layer forward (wk_layer_forward_noalloc) against the fp64 oracle.

Some callers cannot let a library call cudaMalloc: a serving process that gave all
device memory to its own pool allocator, or a latency-critical loop in which
cudaMalloc / cudaFree (which synchronise the device) are not allowed. For them the
library offers one layer whose intermediates live in a fixed device array compiled
into the library. Each case runs the call twice in a row (the array keeps the first
call's contents, which the second must not depend on) and compares both outputs with
the oracle's layer (the Wukong page, section 2.2) on sampled examples: 2e-2 for the
16-bit workloads (bf16, and the same layer in fp16), 1e-4 for the fp32 workload, the
tolerances of the stack tests. This file runs last so that, if it fails, a run that
stops at the first failure has already run every other test; it passes alone in a
fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, max_scaled_err

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 2e-2, "f16": 2e-2}


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _case(name, dtype, batch):
    """Device layer and X in `dtype`, and the same values as host arrays for the oracle."""
    cfg = dict(C.CONFIGS[name], layers=1)
    layer = C.make_layer_dev(cfg, 0)
    X = C.make_x_dev(cfg, batch)
    host = C.make_layer_host(cfg, 0)
    if dtype == "f16":  # the bf16 workload's values rounded to fp16 on the device
        for key in ["Y", "W_L"] + ["W%d" % j for j in range(len(cfg["hidden"]) + 1)]:
            layer[key] = layer[key].to(torch.float16)
            host[key] = layer[key].float().cpu().numpy()  # exact: fp16 values are float32 values
        X = X.to(torch.float16)
        cfg = dict(cfg, dtype="f16")
    return cfg, layer, X, host


@pytest.mark.parametrize("name,dtype,batch,n_sample", [("c1_fp32", "f32", 64, 64), ("c2_bf16", "bf16", 256, 16),
                                                       ("c2_bf16", "f16", 200, 16), ("c5_bf16", "bf16", 128, 8)])
def test_noalloc_layer_matches_oracle_on_two_calls(name, dtype, batch, n_sample):
    cfg, layer, X, host = _case(name, dtype, batch)
    ex = sorted(set([0, 1, batch // 2, batch - 1] + list(np.random.RandomState(3).choice(batch, n_sample - 4,
                                                                                        replace=False))))
    ref = oracle.layer_forward(cfg, host, f64(X[ex]))
    for call in range(2):
        out = torch.full_like(X, float("nan"))
        wk.wk_layer_forward_noalloc(cfg, layer, X, out)
        torch.cuda.synchronize()
        assert wk.wk_device_status() == wk.WK_OK
        got = f64(out)
        assert np.isfinite(got).all()
        err = max_scaled_err(got[ex], ref)
        print("%s %s call %d: max scaled error vs the fp64 oracle %.3g" % (name, dtype, call, err))
        assert err <= TOL[dtype]


def test_noalloc_rejects_batch_beyond_the_static_scratch():
    cfg = dict(C.CONFIGS["c2_bf16"], layers=1)
    layer = C.make_layer_dev(cfg, 0)
    per_example = 2 * (cfg["n"] * cfg["k"] + cfg["n"] * cfg["d"] + max(cfg["hidden"]))
    batch = (32 * 1024 * 1024) // per_example + 64
    X = C.make_x_dev(cfg, batch)
    out = torch.empty_like(X)
    with pytest.raises(wk.WkError) as e:
        wk.wk_layer_forward_noalloc(cfg, layer, X, out)
    assert e.value.status == wk.WK_ERR_INVALID_ARG
