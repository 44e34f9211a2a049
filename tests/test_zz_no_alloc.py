"""The no-allocation one-layer forward (wk_layer_forward_noalloc) against the
stack forward of the same layer.

Some callers cannot let a library call cudaMalloc: a serving process that gave all
device memory to its own pool allocator, or a latency-critical loop in which
cudaMalloc / cudaFree (which synchronise the device) are not allowed. For them the
library offers one layer whose intermediates live in a fixed device array compiled
into the library. This file runs last so that, if it fails, a run that stops at the
first failure has already run every other test; it passes alone in a fresh process
and after the other tests.
"""
import numpy as np
import pytest
import torch

import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, max_scaled_err

pytestmark = pytest.mark.gpu

TOL = 2e-2  # the bf16-workload parity tolerance of the stack tests


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


@pytest.mark.parametrize("name,batch", [("c2_bf16", 256), ("c5_bf16", 128)])
def test_noalloc_layer_matches_stack_forward_on_two_calls(name, batch):
    cfg = dict(C.CONFIGS[name], layers=1)
    layer = C.make_layer_dev(cfg, 0)
    X = C.make_x_dev(cfg, batch)
    h = wk.wk_stack_create(cfg, [layer], max_batch=batch, operand_dtype=cfg["dtype"])
    ref = torch.empty_like(X)
    wk.wk_stack_forward(h, X, ref)
    torch.cuda.synchronize()
    assert wk.wk_stack_sync_status(h) == wk.WK_OK
    wk.wk_stack_destroy(h)
    for call in range(2):
        out = torch.full_like(X, float("nan"))
        wk.wk_layer_forward_noalloc(cfg, layer, X, out)
        torch.cuda.synchronize()
        assert wk.wk_device_status() == wk.WK_OK
        got = f64(out)
        assert np.isfinite(got).all()
        err = max_scaled_err(got, f64(ref))
        print("%s call %d: max scaled difference to the stack forward %.3g" % (name, call, err))
        assert err <= TOL


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
