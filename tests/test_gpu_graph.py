"""A forward captured in a CUDA graph (wk_stack_graph_create / wk_moe_graph_create) and
replayed with wk_graph_launch computes exactly what the eager forward computes (the
same kernels, in the same order), replays repeatably, and reads the input buffer's
contents at replay time."""
import pytest
import torch

import recsys_feature_interaction_b200 as wk
from synth import configs as C

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


@pytest.mark.parametrize("name,batch", [("c2_bf16", 1000), ("c1_fp32", 64), ("c5_bf16", 512)])
def test_stack_graph_matches_eager(name, batch):
    cfg = C.CONFIGS[name]
    layers = [C.make_layer_dev(cfg, l) for l in range(cfg["layers"])]
    h = wk.wk_stack_create(cfg, layers, max_batch=batch)
    try:
        X = C.make_x_dev(cfg, batch)
        ref = torch.empty_like(X)
        wk.wk_stack_forward(h, X, ref)
        out = torch.full_like(X, float("nan"))
        g = wk.wk_stack_graph_create(h, X, out)
        wk.wk_graph_launch(g)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        out.fill_(float("nan"))
        wk.wk_graph_launch(g)
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
        # new contents in the captured input buffer
        X2 = C.make_x_dev(cfg, batch, first_example=batch)
        ref2 = torch.empty_like(X)
        wk.wk_stack_forward(h, X2, ref2)
        X.copy_(X2)
        wk.wk_graph_launch(g)
        torch.cuda.synchronize()
        assert torch.equal(out, ref2)
        assert wk.wk_stack_sync_status(h) == wk.WK_OK
        wk.wk_graph_destroy(g)
    finally:
        wk.wk_stack_destroy(h)


def test_moe_graph_matches_eager():
    cfg = C.MOE_CONFIGS["moe3_c2"]
    batch = 700
    experts = [[C.make_expert_dev(cfg, l, e) for e in range(cfg["experts"])] for l in range(cfg["layers"])]
    gates = [C.make_gate_dev(cfg, l) for l in range(cfg["layers"])]
    h = wk.wk_moe_create(cfg, experts, gates, max_batch=batch)
    try:
        X = C.make_x_dev(cfg, batch)
        ref = torch.empty_like(X)
        wk.wk_moe_forward(h, X, ref)
        out = torch.full_like(X, float("nan"))
        g = wk.wk_moe_graph_create(h, X, out)
        for _ in range(2):
            wk.wk_graph_launch(g)
            torch.cuda.synchronize()
            assert torch.equal(out, ref)
        assert wk.wk_moe_sync_status(h) == wk.WK_OK
        wk.wk_graph_destroy(g)
    finally:
        wk.wk_moe_destroy(h)
