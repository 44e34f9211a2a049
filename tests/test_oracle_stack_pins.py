"""Pins of the oracle's layer composition: oracle.stack_forward (the Wukong page, section
2.2: layers are stacked, each layer's output is the next layer's input; section 2.3: the
depth l is a scaling knob) and oracle.moe_forward (the Kunlun page, section 2.3: the
Wukong-MoE layer, stacked the same way).

Every expected value is a closed form evaluated without the oracle: each layer is chosen
so that its output is written through torch's LayerNorm and a numpy product in the other
association of the FM, X (X^T Y). The layers of a stack differ from one another (their
W_L select different rows, their constant FMB rows and LayerNorm affines differ, one layer
crosses features through the FM), so a slip in the chaining fails: feeding X to every layer
instead of the previous layer's output, taking layer 0's weights for every layer, skipping
or repeating a layer, or running the layers out of order. Each test also checks that those
wrong compositions give visibly different outputs, so the pin discriminates.
"""
import numpy as np
import torch

import oracle

# n * k == n_f * d, so one Linear of the identity can carry the FM output straight into
# the FMB rows (the cfg is shared by every layer of a stack: one Linear, no hidden layer)
N, D, K, NF, NL = 6, 3, 2, 4, 2


def _cfg(layers, **kw):
    return dict(n=N, d=D, k=K, n_f=NF, n_l=NL, hidden=[], layers=layers, **kw)


def _ln_rows(x, g=None, b=None, eps=1e-5):
    t = torch.tensor(np.asarray(x, np.float64))
    G = None if g is None else torch.tensor(np.asarray(g, np.float64))
    B = None if b is None else torch.tensor(np.asarray(b, np.float64))
    return torch.nn.functional.layer_norm(t, (t.shape[-1],), G, B, eps).numpy()


def _zero_layer():
    return {"Y": np.zeros((N, K), np.float32), "W0": np.zeros((NF * D, N * K), np.float32),
            "b0": np.zeros(NF * D, np.float32), "fmb_gamma": np.ones(N * K, np.float32),
            "fmb_beta": np.zeros(N * K, np.float32), "W_L": np.zeros((NL, N), np.float32),
            "out_gamma": np.ones(D, np.float32), "out_beta": np.zeros(D, np.float32)}


def _const_layer(rng, sel, beta_sum=None):
    """FMB rows constant (all FMB weights zero but the Linear's bias c), W_L picks rows sel
    of the layer input, random output LayerNorm affine (beta summing to beta_sum if given)."""
    w = _zero_layer()
    w["b0"] = rng.uniform(-2.0, 2.0, NF * D).astype(np.float32)
    w["W_L"] = np.eye(N, dtype=np.float32)[list(sel)]
    w["out_gamma"] = rng.uniform(0.5, 1.5, D).astype(np.float32)
    beta = rng.uniform(-1.0, 1.0, D)
    if beta_sum is not None:
        w["out_gamma"][:] = 1.0
        beta = beta - beta.mean() + beta_sum / D
        # float32 storage: put the rounding of the sum on the last entry
        beta = beta.astype(np.float32)
        beta[-1] = np.float32(beta_sum - float(np.sum(beta[:-1].astype(np.float64))))
    w["out_beta"] = np.asarray(beta, np.float32)
    return w


def _fm_layer(rng, sel):
    """FMB rows = reshape(LN(flatten(X X^T Y)) * g + b) through one identity Linear."""
    w = _zero_layer()
    w["Y"] = rng.randn(N, K).astype(np.float32)
    w["W0"] = np.eye(N * K, dtype=np.float32)
    w["fmb_gamma"] = rng.uniform(0.5, 1.5, N * K).astype(np.float32)
    w["fmb_beta"] = (0.3 * rng.randn(N * K)).astype(np.float32)
    w["W_L"] = np.eye(N, dtype=np.float32)[list(sel)]
    w["out_gamma"] = rng.uniform(0.5, 1.5, D).astype(np.float32)
    w["out_beta"] = rng.uniform(-1.0, 1.0, D).astype(np.float32)
    return w


def _closed_layer(w, X):
    """The layer's output in closed form, for the two kinds of layer above."""
    f64 = lambda a: np.asarray(a, np.float64)
    out = np.empty_like(X)
    for e in range(X.shape[0]):
        x = X[e]
        if np.any(w["W0"]):  # the FM layer: the identity Linear passes the FMB LayerNorm through
            F = x @ (x.T @ f64(w["Y"]))
            fmb = _ln_rows(F.reshape(-1), w["fmb_gamma"], w["fmb_beta"]).reshape(NF, D)
        else:
            fmb = f64(w["b0"]).reshape(NF, D)
        lcb = f64(w["W_L"]) @ x  # a row selection: exact
        out[e] = _ln_rows(np.concatenate([fmb, lcb]) + x, w["out_gamma"], w["out_beta"])
    return out


def _chain(ws, X):
    h = X
    for w in ws:
        h = _closed_layer(w, h)
    return h


def _far(a, b):
    return float(np.max(np.abs(a - b))) > 0.1


def test_stack_forward_chains_distinct_layers():
    rng = np.random.RandomState(21)
    ws = [_fm_layer(rng, [5, 0]), _const_layer(rng, [1, 3]), _const_layer(rng, [2, 2])]
    X = rng.randn(4, N, D)
    got = oracle.stack_forward(_cfg(3), lambda l: ws[l], X)
    want = _chain(ws, X)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-11), np.max(np.abs(got - want))
    # the wrong compositions this pin must tell apart from the right one
    wrong = {
        "X fed to every layer": _closed_layer(ws[2], X),
        "layer 0's weights everywhere": _chain([ws[0]] * 3, X),
        "last layer skipped": _chain(ws[:2], X),
        "first layer repeated": _chain([ws[0], ws[0], ws[1]], X),
        "layers reversed": _chain(ws[::-1], X),
    }
    for name, v in wrong.items():
        assert _far(v, want), name


def test_stack_forward_one_layer_per_call_matches_depth():
    """Depth is the number of layers the config names: a 2-layer call is the first two
    layers of the 3-layer chain, not all three and not one."""
    rng = np.random.RandomState(22)
    ws = [_const_layer(rng, [4, 1]), _fm_layer(rng, [0, 2]), _const_layer(rng, [3, 5])]
    X = rng.randn(3, N, D)
    got = oracle.stack_forward(_cfg(2), lambda l: ws[l], X)
    assert np.allclose(got, _chain(ws[:2], X), rtol=1e-11, atol=1e-11)
    assert _far(got, _chain(ws, X)) and _far(got, _chain(ws[:1], X))


def test_moe_forward_chains_layers_and_gates_on_the_layer_input():
    """Two MoE layers of three experts each. Layer 0's gate selects expert 1 by its bias.
    Layer 1's gate reads the sum of input row 0 (weight 300 for expert 2, 0 for the others):
    layer 0's output rows are LayerNorm outputs with gamma = 1 and beta summing to 1, so the
    sum is 1 and expert 2 wins; the input X has row sums of -1, which would give experts 0
    and 1 half each. So the result is expert (1, 2)'s layer of expert (0, 1)'s layer of X,
    exactly (the other gate weights underflow to 0)."""
    rng = np.random.RandomState(23)
    sels = [[[0, 1], [2, 4], [5, 3]], [[1, 1], [4, 0], [3, 2]]]
    experts = [[_const_layer(rng, s, beta_sum=1.0 if (l, e) == (0, 1) else None) for e, s in enumerate(sels[l])]
               for l in range(2)]
    experts[1][0] = _fm_layer(rng, sels[1][0])
    nd = N * D
    gates = [{"W_g": np.zeros((3, nd), np.float32), "b_g": np.array([0.0, 800.0, 0.0], np.float32)},
             {"W_g": np.zeros((3, nd), np.float32), "b_g": np.zeros(3, np.float32)}]
    gates[1]["W_g"][2, :D] = 300.0
    X = rng.randn(3, N, D)
    X[:, 0, :] += (-1.0 - X[:, 0, :].sum(axis=1, keepdims=True)) / D  # row 0 sums to -1
    cfg = _cfg(2, experts=3)
    got = oracle.moe_forward(cfg, lambda l, e: experts[l][e], lambda l: gates[l], X)
    h1 = _closed_layer(experts[0][1], X)
    assert np.allclose(h1[:, 0, :].sum(axis=1), 1.0, rtol=0, atol=1e-12)
    want = _closed_layer(experts[1][2], h1)
    assert np.allclose(got, want, rtol=1e-11, atol=1e-11), np.max(np.abs(got - want))
    wrong = {
        "X fed to layer 1": _closed_layer(experts[1][2], X),
        "layer 1 gate read from X": 0.5 * (_closed_layer(experts[1][0], h1) + _closed_layer(experts[1][1], h1)),
        "layer 0's experts reused": _closed_layer(experts[0][2], h1),
        "one layer only": h1,
    }
    for name, v in wrong.items():
        assert _far(v, want), name
