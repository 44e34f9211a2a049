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


def test_streamed_host_forward_matches_the_device_forward():
    # a serving loop: each call enqueues its input copy, forward and output copy; the
    # previous call's result is waited for after the next call is issued, with two
    # alternating pairs of page-locked host buffers and ragged batch sizes
    cfg = C.CONFIGS["c2_bf16"]
    st = DevStack("c2_bf16")
    try:
        B = cfg["batch"]
        sizes = [B, 1000, B, 17, 2048, B]
        xs = [C.make_x_dev(cfg, B, first_example=7 * B * j) for j in range(len(sizes))]
        want = [st.run(x[:nb].contiguous()).cpu() for x, nb in zip(xs, sizes)]
        xh = [torch.empty_like(xs[0], device="cpu").pin_memory() for _ in range(2)]
        oh = [torch.empty_like(xs[0], device="cpu").pin_memory() for _ in range(2)]
        got, prev = [], None
        for j, nb in enumerate(sizes):
            xh[j % 2][:nb].copy_(xs[j][:nb].cpu())
            t = wk.wk_stack_forward_host_async(st.h, xh[j % 2], oh[j % 2], batch=nb)
            if prev is not None:
                wk.wk_stack_host_wait(st.h, prev[0])
                got.append(oh[prev[1] % 2][:sizes[prev[1]]].clone())
            prev = (t, j)
        with pytest.raises(wk.WkError):
            wk.wk_stack_host_wait(st.h, prev[0] + 1)  # not issued yet
        wk.wk_stack_host_wait(st.h)
        got.append(oh[prev[1] % 2][:sizes[prev[1]]].clone())
        assert wk.wk_stack_sync_status(st.h) == wk.WK_OK
        for j, (g, w) in enumerate(zip(got, want)):
            assert torch.equal(g, w), "call %d" % j
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
        # per layer one front kernel (input LayerNorm, FM + LayerNorm, LCB, residual) and the
        # MLP Linears; one output LayerNorm for the stack
        assert t["front"][1] == cfg["layers"] and t["mlp_gemm"][1] == cfg["layers"] * m
        assert t["res_ln"][1] == 1 and t["fm_ln"][1] == 0 and t["lcb"][1] == 0 and t["convert"][1] == 0
        assert all(ms > 0 for ms, count in t.values() if count)
    finally:
        st.close()


def test_parity_c4_bf16_full_size():
    _parity("c4_bf16", 16)


@pytest.mark.parametrize("name,batch", [("c2_bf16", 100), ("c2_bf16", 7), ("c3_bf16", 149), ("c5_bf16", 37),
                                        ("c4_bf16", 3)])
def test_parity_small_and_ragged_batches(name, batch):
    """Batches below one CTA per SM, not a multiple of the grid, and at most one 128-row MLP
    tile (the one-CTA GEMM with its reduce-add epilogue): every example against the oracle."""
    cfg = C.CONFIGS[name]
    st = DevStack(name, max_batch=batch)
    try:
        X = C.make_x_dev(cfg, batch)
        out = st.run(X)
        ex = list(range(batch)) if batch <= 16 else _sample(batch, 16)
        got = f64(out[ex])
        assert np.isfinite(got).all()
        err = max_scaled_err(got, _oracle(cfg, ex))
        print("%s batch %d: max |gpu-ref|/(1+|ref|) = %.3g" % (name, batch, err))
        assert err <= TOL[cfg["dtype"]]
    finally:
        st.close()
        torch.cuda.empty_cache()


@pytest.mark.parametrize("what", ["input", "hidden"])
def test_fp16_overflow_is_reported(what):
    """The default 16-bit path keeps its intermediates in fp16 (range |v| <= 65504), where the
    pages' bf16 has the range of fp32. A value past that range must come back as
    WK_ERR_NONFINITE from the status call, not as silent inf / NaN in the output: an input
    scaled by 1e5 (representable in the caller's bf16, not in fp16), or a first Linear scaled
    by 1e5 (its hidden activations overflow). A normal forward afterwards reports WK_OK."""
    cfg = dict(C.CONFIGS["c2_bf16"], layers=1)
    layer = C.make_layer_dev(cfg, 0)
    X = C.make_x_dev(cfg, 64)
    if what == "input":
        Xb = (X.float() * 1e5).to(X.dtype)
        assert torch.isfinite(Xb).all()
        layers = [layer]
    else:
        Xb = X
        layers = [dict(layer, W0=(layer["W0"].float() * 1e5).to(layer["W0"].dtype))]
    h = wk.wk_stack_create(cfg, layers, max_batch=64)
    try:
        out = torch.empty_like(X)
        wk.wk_stack_forward(h, Xb, out)
        assert wk.wk_stack_sync_status(h) == wk.WK_ERR_NONFINITE
        assert "non-finite" in wk.wk_status_string(wk.WK_ERR_NONFINITE)
    finally:
        wk.wk_stack_destroy(h)
    h = wk.wk_stack_create(cfg, [layer], max_batch=64)
    try:
        out = torch.empty_like(X)
        wk.wk_stack_forward(h, X, out)
        assert wk.wk_stack_sync_status(h) == wk.WK_OK
        assert torch.isfinite(out.float()).all()
    finally:
        wk.wk_stack_destroy(h)


def test_parity_fp16_caller_stack():
    """A caller whose tensors are fp16 (the operand type): the first layer's front copies the
    input into the operand layout without a conversion, and the output is written in fp16.
    The bf16 workload's values rounded to fp16 on the device; the oracle reads the same fp16
    values (exact in float32)."""
    cfg = dict(C.CONFIGS["c2_bf16"], dtype="f16")
    batch = 300
    host_layers, dev_layers = [], []
    for l in range(cfg["layers"]):
        d = C.make_layer_dev(C.CONFIGS["c2_bf16"], l)
        h = C.make_layer_host(C.CONFIGS["c2_bf16"], l)
        for key in ["Y", "W_L"] + ["W%d" % j for j in range(len(cfg["hidden"]) + 1)]:
            d[key] = d[key].to(torch.float16)
            h[key] = d[key].float().cpu().numpy()
        dev_layers.append(d)
        host_layers.append(h)
    X = C.make_x_dev(C.CONFIGS["c2_bf16"], batch).to(torch.float16)
    h = wk.wk_stack_create(cfg, dev_layers, max_batch=batch)
    try:
        out = torch.empty_like(X)
        wk.wk_stack_forward(h, X, out)
        torch.cuda.synchronize()
        assert wk.wk_stack_sync_status(h) == wk.WK_OK
        assert out.dtype == torch.float16
        ex = _sample(batch, 16)
        got = f64(out[ex])
        ref = oracle.stack_forward(cfg, lambda l: host_layers[l], f64(X[ex]))
        err = max_scaled_err(got, ref)
        print("c2 shape, fp16 caller: max |gpu-ref|/(1+|ref|) = %.3g" % err)
        assert err <= TOL["bf16"]
    finally:
        wk.wk_stack_destroy(h)
