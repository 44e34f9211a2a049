"""Backward pass of the stack on the GPU (wk_stack_backward) against the fp64 oracle
(oracle.layer_backward chained over the layers, each layer's input from the C forward).

The forward is the Wukong page's layer (section 2.2); the backward is its derivative by the
chain rule. Inputs: the seeded workloads' weights (bf16), X from the generator, dOut ~ N(0, 1).
Every gradient tensor (dX and, per layer, Y, W_j, b_j, the FMB LayerNorm's gamma and beta, W_L
and the output LayerNorm's gamma and beta) is compared with the oracle.

Tolerance: max |gpu - ref| <= 2e-2 * max |ref| per tensor (the tensor's largest entry sets
the scale: weight gradients are sums over the batch, so a per-entry (1 + |ref|) scale would
not be uniform across them). The GPU's operands and MLP gradients are fp16, accumulation fp32.

The ReLU derivative is a decision taken in floating point: where a pre-activation lies within
rounding of 0, the GPU (fp16 operands, fp32 sums) and the fp64 oracle may take different,
equally valid, subgradients, and on a small batch one such unit moves the upstream gradients
by percents. The cases are therefore built so that no gate is near its threshold, and
everything is compared in full against the oracle's exact gates (pre-activation > 0 in
float64). Two constructions: the workload's own weights with the hidden bias of each unit
whose pre-activation comes within 5e-3 rms of 0 in some example moved just far enough to clear
that band (at every layer, the layer's input taken from the oracle's forward; asserted to be
few units), and one layer with its hidden biases moved to +-5 times the spread of its
pre-activations, where no pre-activation is near 0 (asserted): the 4-layer shape on 8
examples, and the 2-layer shape on 256 examples, where both MLP gradient GEMMs (batch and
hidden width above 128) run on the CTA-pair kernel with operands read MN-major instead of
transposed.
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


def _check(name, got, ref):
    got = got.double().cpu().numpy() if isinstance(got, torch.Tensor) else got
    assert np.isfinite(got).all(), name
    scale = max(np.max(np.abs(ref)), 1e-30)
    return float(np.max(np.abs(got - ref)) / scale)


REL = 5e-3  # a pre-activation this close to 0 (times its rms) counts as near the threshold


def _near_zero_units(cfg, w, X, rel=REL):
    """Per hidden Linear j: the units whose pre-activation lies within rel * rms of 0 in
    some example (the oracle's float64 forward)."""
    _, c = oracle.layer_forward_np(cfg, w, X)
    out = {}
    for j, z in enumerate(c["zs"][:-1]):
        rms = np.sqrt(np.mean(z * z))
        out[j] = np.any(np.abs(z) < rel * rms, axis=0)
    return out


def _clear_band_shift(z, band):
    """The smallest shift s (by magnitude) such that no value of z + s lies in (-band, band)."""
    cands = sorted({0.0} | {float(v) for zi in z for v in (band - zi, -band - zi)}, key=abs)
    for s in cands:
        if np.all(np.abs(z + s) >= band * (1.0 - 1e-9)):  # a boundary candidate lands on the band
            return s
    raise AssertionError("no shift clears the band")


def _clear_near_zero_gates(cfg, host_w, dev_w, X):
    """Every layer in order (its input from the oracle's forward of the layers before): the
    hidden bias of each unit with a pre-activation within REL * rms of 0 in some example moves
    by the smallest amount that puts all of that unit's pre-activations at least 1.5 * REL * rms
    away from 0. Returns the number of units moved per layer and Linear."""
    m = len(cfg["hidden"]) + 1
    moved = []
    x = X
    for l, w in enumerate(host_w):
        for j in range(m - 1):
            if w.get("b%d" % j) is None:
                w["b%d" % j] = np.zeros(cfg["hidden"][j], dtype=np.float32)
            _, c = oracle.layer_forward_np(cfg, w, x)
            z = c["zs"][j]
            rms = float(np.sqrt(np.mean(z * z)))
            near = np.any(np.abs(z) < REL * rms, axis=0)
            b = w["b%d" % j].astype(np.float32).copy()
            for u in np.nonzero(near)[0]:
                b[u] = np.float32(b[u] + _clear_band_shift(z[:, u], 1.5 * REL * rms))
            w["b%d" % j] = b
            dev_w[l]["b%d" % j] = to_dev(b)
            moved.append(int(near.sum()))
        assert not any(v.any() for v in _near_zero_units(cfg, w, x).values()), l
        x = oracle.layer_forward(dict(cfg, layers=1), w, x)
    return moved


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
    Xh = C.to_f64(C.make_x_host(cfg, list(range(batch))))
    if shift:
        assert layers == 1
        _shift_hidden_biases(cfg, host_w, dev_layers, Xh, 141)
    else:
        moved = _clear_near_zero_gates(cfg, host_w, dev_layers, Xh)
        assert all(v <= 0.1 * max(cfg["hidden"]) for v in moved), moved  # most units keep their bias
    h = wk.wk_stack_create(cfg, dev_layers, max_batch=batch)
    X = C.make_x_dev(cfg, batch)
    dOut_h = host_normal((batch, cfg["n"], cfg["d"]), 131, dtype="f32")
    dOut = to_dev(dOut_h)
    dX = torch.full_like(dOut, float("nan"))
    grads = _grads_dev(cfg, dims)
    wk.wk_stack_backward(h, X, dOut, dX, grads)
    assert wk.wk_stack_sync_status(h) == wk.WK_OK
    # the oracle: layer inputs from the C forward, then the layers' backwards, last first;
    # the ReLU gates are the oracle's own (pre-activation > 0 in float64)
    xs = [Xh]
    for l in range(layers - 1):
        xs.append(oracle.layer_forward(dict(cfg, layers=1), host_w[l], xs[-1]))
    up = f64(dOut_h)
    errs = {}
    for l in range(layers - 1, -1, -1):
        # no gate near its threshold at any layer: compared in full
        assert not any(v.any() for v in _near_zero_units(cfg, host_w[l], xs[l]).values()), l
        up, g = oracle.layer_backward(cfg, host_w[l], xs[l], up)
        gd = grads[l]
        for key, ref in g.items():
            if key[0] == "W" and key != "W_L":
                got = gd["W"][int(key[1:])]
            elif key[0] == "b" and key[1:].isdigit():
                got = gd["b"][int(key[1:])]
            else:
                got = gd[key]
            errs["%d.%s" % (l, key)] = _check(key, got, ref)
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
