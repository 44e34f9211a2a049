"""The prediction head after the Wukong stack (Wukong page, section 2.2: the stacked
layers cross the features, an MLP then produces the prediction; reading: flatten,
Linear + ReLU layers, one logit, sigmoid) through wk_stack_predict, against the fp64
oracle (stack, then head) on sampled examples.

Tolerance: the logit as the stack output, max |gpu - ref| / (1 + |ref|) <= 2e-2; the
probability (a 1-Lipschitz/4 function of the logit) within 1e-2 absolute.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _sample(batch, count, seed=0):
    rng = np.random.RandomState(seed)
    fixed = [0, 1, batch // 2, batch - 1]
    rest = rng.choice(np.arange(2, batch - 1), size=max(0, count - len(fixed)), replace=False).tolist()
    return sorted(set(fixed + rest))[:count]


@pytest.mark.parametrize("name,hidden,n_sample,batch", [("c2_bf16", None, 128, None), ("c2_bf16", [], 64, 1000),
                                                        ("c2_bf16", [264], 64, 333), ("c3_bf16", None, 8, 4096)])
def test_predict_parity(name, hidden, n_sample, batch):
    cfg = C.CONFIGS[name]
    B = batch or cfg["batch"]
    layers = [C.make_layer_dev(cfg, l) for l in range(cfg["layers"])]
    h = wk.wk_stack_create(cfg, layers, max_batch=B)
    try:
        head = C.make_head_dev(cfg, hidden)
        wk.wk_stack_set_head(h, head)
        X = C.make_x_dev(cfg, B)
        logit = torch.full((B,), float("nan"), device="cuda")
        prob = torch.full((B,), float("nan"), device="cuda")
        wk.wk_stack_predict(h, X, logit, prob)
        torch.cuda.synchronize()
        assert wk.wk_stack_sync_status(h) == wk.WK_OK
        ex = _sample(B, n_sample)
        Xh = C.to_f64(C.make_x_host(cfg, ex))
        xl = oracle.stack_forward(cfg, lambda l: C.make_layer_host(cfg, l), Xh)
        ref_logit, ref_p = oracle.top_mlp_forward(C.make_head_host(cfg, hidden), xl)
        got = logit[ex].double().cpu().numpy()
        gotp = prob[ex].double().cpu().numpy()
        assert np.isfinite(got).all()
        err = float(np.max(np.abs(got - ref_logit) / (1 + np.abs(ref_logit))))
        print("%s head %s: max logit error %.3g (|logit| up to %.2f), max prob error %.3g"
              % (name, hidden, err, np.max(np.abs(ref_logit)), np.max(np.abs(gotp - ref_p))))
        assert err <= 2e-2
        assert np.max(np.abs(gotp - ref_p)) <= 1e-2
        assert np.allclose(gotp, 1.0 / (1.0 + np.exp(-got)), rtol=0, atol=1e-6)
        # the stack output itself is unchanged by the head (predict then forward)
        out = torch.empty_like(X)
        wk.wk_stack_forward(h, X, out)
        torch.cuda.synchronize()
        assert np.max(np.abs(out[ex].double().cpu().numpy() - xl) / (1 + np.abs(xl))) <= 2e-2
    finally:
        wk.wk_stack_destroy(h)
        torch.cuda.empty_cache()


def test_predict_without_head_is_an_argument_error():
    cfg = C.CONFIGS["c2_bf16"]
    layers = [C.make_layer_dev(cfg, l) for l in range(cfg["layers"])]
    h = wk.wk_stack_create(cfg, layers, max_batch=64)
    try:
        X = C.make_x_dev(cfg, 64)
        logit = torch.empty(64, device="cuda")
        with pytest.raises(wk.WkError) as ei:
            wk.wk_stack_predict(h, X, logit)
        assert ei.value.status == wk.WK_ERR_INVALID_ARG
    finally:
        wk.wk_stack_destroy(h)
