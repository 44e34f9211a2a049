"""Backward pass of the stack on the GPU (wk_stack_backward) against the fp64 oracle
(oracle.layer_backward chained over the layers, each layer's input from the C forward).

The forward is the Wukong page's layer (section 2.2); the backward is its derivative by the
chain rule. Inputs: the seeded workloads' weights (bf16), X from the generator, dOut ~ N(0, 1).
Every gradient tensor (dX and, per layer, Y, W_j, b_j, the FMB LayerNorm's gamma and beta, W_L
and the output LayerNorm's gamma and beta) is compared with the oracle.

Tolerance: max |gpu - ref| <= 2e-2 * max |ref| per tensor (the tensor's largest entry sets
the scale: weight gradients are sums over the batch, so a per-entry (1 + |ref|) scale would
not be uniform across them). The GPU's operands and MLP gradients are fp16, accumulation fp32.

The ReLU derivative is a decision taken in floating point, so the oracle takes it in the
kernels' precision (oracle.relu_gates_fp16: the forward rounded where the fp16 path stores
it). Only the GPU's fp32 summation order then separates the two, so a gate can still differ
where a pre-activation is within about 1e-4 of zero, and on a small batch such a difference
moves the upstream gradients by percents (both are valid subgradients). Two cases therefore:
the workload's own weights (deeper layers: units with |z| < 2e-3 rms(z) in some example are
left out of their own W_j rows and b_j, and must be few), and one layer with its hidden biases
moved to +-5 times the spread of its pre-activations, where no pre-activation is near 0
(asserted) and everything is compared in full: the 4-layer shape on 8 examples, and the 2-layer
shape on 256 examples, where both MLP gradient GEMMs (batch and hidden width above 128) run on
the CTA-pair kernel with operands read MN-major instead of transposed.
"""
import numpy as np
import pytest
import torch

import oracle
import recsys_feature_interaction_b200 as wk
from synth import configs as C
from tests.gpu_util import f64, host_normal, to_dev

pytestmark = pytest.mark.gpu

TOL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _lib(cuda_device):
    from recsys_feature_interaction_b200 import build
    build.build()
    wk.lib()


def _grads_dev(cfg, dims):
    L = cfg["layers"]
    n, d, k, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_l"]
    z = lambda *s: torch.full(s, float("nan"), dtype=torch.float32, device="cuda")
    return [{"Y": z(n, k), "W": [z(dims[j + 1], dims[j]) for j in range(len(dims) - 1)],
             "b": [z(dims[j + 1]) for j in range(len(dims) - 1)], "fmb_gamma": z(n * k), "fmb_beta": z(n * k),
             "W_L": z(n_l, n), "out_gamma": z(d), "out_beta": z(d)} for _ in range(L)]


def _check(name, got, ref, keep=None):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert np.isfinite(got).all(), name
    scale = max(np.max(np.abs(ref)), 1e-30)
    diff = np.abs(got - ref)
    if keep is not None:
        diff = diff[keep]
    return float(np.max(diff) / scale)


def _unambiguous_units(cfg, w, X, rel=2e-3):
    """Per hidden Linear j: the units whose pre-activation is away from 0 in every example."""
    _, c = oracle.layer_forward_np(cfg, w, X)
    out = {}
    for j, z in enumerate(c["zs"][:-1]):
        rms = np.sqrt(np.mean(z * z))
        out[j] = np.all(np.abs(z) >= rel * rms, axis=0)
    return out


def _shift_hidden_biases(cfg, host_w, dev_w, X, seed):
    """One layer: each hidden Linear's bias set to +-5 times the spread of its pre-activation
    without bias (seeded signs, measured on the oracle's forward Linear by Linear): every ReLU
    pre-activation is then far from 0, so no gate is ambiguous."""
    m = len(cfg["hidden"]) + 1
    for j in range(m - 1):
        host_w[0]["b%d" % j] = np.zeros(cfg["hidden"][j], dtype=np.float32)
        _, c = oracle.layer_forward_np(cfg, host_w[0], X)
        spread = float(np.std(c["zs"][j]))
        sign = np.where(np.random.RandomState(seed + j).rand(cfg["hidden"][j]) < 0.5, -1.0, 1.0)
        b = (5.0 * spread * sign).astype(np.float32)
        host_w[0]["b%d" % j] = b
        dev_w[0]["b%d" % j] = to_dev(b)


@pytest.mark.parametrize("name,batch,layers,shift", [("c2_bf16", 16, 2, False), ("c3_bf16", 8, 1, True),
                                                     ("c2_bf16", 256, 1, True)])
def test_stack_backward_against_oracle(name, batch, layers, shift):
    cfg = dict(C.CONFIGS[name], layers=layers)
    dims = C.mlp_dims(cfg)
    dev_layers = [C.make_layer_dev(cfg, l) for l in range(layers)]
    host_w = [C.make_layer_host(cfg, l) for l in range(layers)]
    if shift:
        assert layers == 1
        _shift_hidden_biases(cfg, host_w, dev_layers, C.to_f64(C.make_x_host(cfg, list(range(batch)))), 141)
    h = wk.wk_stack_create(cfg, dev_layers, max_batch=batch)
    X = C.make_x_dev(cfg, batch)
    dOut_h = host_normal((batch, cfg["n"], cfg["d"]), 131, dtype="f32")
    dOut = to_dev(dOut_h)
    dX = torch.full_like(dOut, float("nan"))
    grads = _grads_dev(cfg, dims)
    wk.wk_stack_backward(h, X, dOut, dX, grads)
    assert wk.wk_stack_sync_status(h) == wk.WK_OK
    # the oracle: layer inputs from the C forward, then the layers' backwards, last first
    Xh = C.to_f64(C.make_x_host(cfg, list(range(batch))))
    xs = [Xh]
    for l in range(layers - 1):
        xs.append(oracle.layer_forward(dict(cfg, layers=1), host_w[l], xs[-1]))
    up = f64(dOut_h)
    errs = {}
    for l in range(layers - 1, -1, -1):
        keep = _unambiguous_units(cfg, host_w[l], xs[l]) if l > 0 else {}
        for j, kj in keep.items():
            assert kj.mean() >= 0.9, (l, j, kj.mean())
        if shift:  # no gate near its threshold: compared in full
            assert all(kj.all() for kj in _unambiguous_units(cfg, host_w[l], xs[l], 1e-2).values())
            keep = {}
        gates = oracle.relu_gates_fp16(cfg, host_w[l], xs[l])
        up, g = oracle.layer_backward(cfg, host_w[l], xs[l], up, gates=gates)
        gd = grads[l]
        for key, ref in g.items():
            kk = None
            if key[0] == "W" and key != "W_L":
                got = gd["W"][int(key[1:])]
                kk = keep.get(int(key[1:]))
            elif key[0] == "b" and key[1:].isdigit():
                got = gd["b"][int(key[1:])]
                kk = keep.get(int(key[1:]))
            else:
                got = gd[key]
            errs["%d.%s" % (l, key)] = _check(key, got, ref, kk)
    errs["dX"] = _check("dX", dX, up)
    worst = max(errs, key=errs.get)
    print(name, "worst", worst, "%.2e" % errs[worst], {k: "%.1e" % v for k, v in sorted(errs.items())})
    assert errs[worst] <= TOL, (worst, errs[worst])
    wk.wk_stack_destroy(h)


def test_backward_rejects_unsupported_batches():
    cfg = dict(C.CONFIGS["c2_bf16"], layers=1)
    dims = C.mlp_dims(cfg)
    h = wk.wk_stack_create(cfg, [C.make_layer_dev(cfg, 0)], max_batch=16)
    X = C.make_x_dev(cfg, 12)
    dOut = torch.zeros((12, cfg["n"], cfg["d"]), dtype=torch.float32, device="cuda")
    with pytest.raises(wk.WkError) as ei:
        wk.wk_stack_backward(h, X, dOut, torch.empty_like(dOut), _grads_dev(cfg, dims), batch=12)
    assert ei.value.status == wk.WK_ERR_UNSUPPORTED
    wk.wk_stack_destroy(h)


def test_layer_events_mark_final_gradients():
    """wk_stack_backward with per-layer events: the gradients (written into the flat per-layer
    buffers a data-parallel step all-reduces) match those of the call without events (bit
    for bit for dX; the batch sums use atomic adds, whose order varies, so those to 1e-4),
    and a second stream that waits on layer l's event copies exactly layer l's final
    gradients while the backward of the layers below runs."""
    from recsys_feature_interaction_b200 import replicas

    cfg = dict(C.CONFIGS["c2_bf16"], layers=2)
    dims = C.mlp_dims(cfg)
    L, batch = cfg["layers"], 16
    h = wk.wk_stack_create(cfg, [C.make_layer_dev(cfg, l) for l in range(L)], max_batch=batch)
    X = C.make_x_dev(cfg, batch)
    dOut = to_dev(host_normal((batch, cfg["n"], cfg["d"]), 133, dtype="f32"))
    dX0, dX1 = torch.empty_like(dOut), torch.empty_like(dOut)
    ref = replicas.GradBuckets(cfg["n"], cfg["d"], cfg["k"], cfg["n_l"], dims, L, device="cuda")
    wk.wk_stack_backward(h, X, dOut, dX0, ref.grads)
    got = replicas.GradBuckets(cfg["n"], cfg["d"], cfg["k"], cfg["n_l"], dims, L, device="cuda")
    evs = [torch.cuda.Event() for _ in range(L)]
    side = torch.cuda.Stream()
    copies = [torch.empty_like(f) for f in got.flats]
    main = torch.cuda.current_stream()
    wk.wk_stack_backward(h, X, dOut, dX1, got.grads, layer_events=evs, stream=main)
    for l in range(L - 1, -1, -1):
        side.wait_event(evs[l])
        with torch.cuda.stream(side):
            copies[l].copy_(got.flats[l])
    torch.cuda.synchronize()
    assert wk.wk_stack_sync_status(h) == wk.WK_OK
    assert all(e.query() for e in evs)
    assert torch.equal(dX0, dX1)
    for l in range(L):
        assert torch.isfinite(ref.flats[l]).all()
        scale = float(ref.flats[l].abs().max())
        assert torch.allclose(got.flats[l], ref.flats[l], rtol=1e-4, atol=1e-5 * scale), l
        assert torch.equal(copies[l], got.flats[l]), l
    with pytest.raises(ValueError):
        wk.wk_stack_backward(h, X, dOut, dX1, got.grads, layer_events=evs[:1])
    wk.wk_stack_destroy(h)
