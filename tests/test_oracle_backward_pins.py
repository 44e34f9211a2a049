"""Pins of the backward-pass oracle (gradients of one Wukong layer; the pages give no
backward, so it is derived from the forward of the Wukong page, section 2.2, by the chain
rule).

Facts that do not come from the oracle's own derivation: central finite differences of the
scalar L = sum(dOut * forward) with respect to every input and parameter tensor (several
entries each, on three small layers: one, two and three Linears, bf16 and float weights),
agreement of the oracle's numpy forward with the C forward (layer_forward), linearity in
dOut, and a ReLU gate that is closed for every example (its unit's incoming weights get no
gradient). A dropped term of the LayerNorm backward, a missing transpose of X X^T, the
residual or the concat order wrong, or a ReLU derivative on the last Linear fails one of them.
"""
import numpy as np
import pytest

import oracle
import synth


def _bf16(a):
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((u + 0x7FFF + ((u >> 16) & 1)) >> 16).astype(np.uint16)


def _layer(cfg, seed, bf16=False):
    rng = np.random.RandomState(seed)
    n, d, k, n_f, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_f"], cfg["n_l"]
    dims = [n * k] + list(cfg["hidden"]) + [n_f * d]
    w = {"Y": rng.randn(n, k) / np.sqrt(n), "W_L": rng.randn(n_l, n) / np.sqrt(n),
         "fmb_gamma": 1 + 0.2 * rng.randn(n * k), "fmb_beta": 0.1 * rng.randn(n * k),
         "out_gamma": 1 + 0.2 * rng.randn(d), "out_beta": 0.1 * rng.randn(d)}
    for j in range(len(dims) - 1):
        w["W%d" % j] = rng.randn(dims[j + 1], dims[j]) / np.sqrt(dims[j])
        w["b%d" % j] = 0.1 * rng.randn(dims[j + 1])
    out = {}
    for key, v in w.items():
        v = v.astype(np.float32)
        out[key] = _bf16(v) if (bf16 and key[0] in "YW") else v
    return out


CASES = [
    (dict(n=4, d=4, k=2, n_f=2, n_l=2, hidden=[]), 1, False),
    (dict(n=4, d=8, k=3, n_f=3, n_l=1, hidden=[6]), 2, True),
    (dict(n=6, d=4, k=2, n_f=2, n_l=4, hidden=[5, 7]), 3, False),
]


def _as_f64(w):
    return {k: (synth.bf16_bits_to_f64(v).reshape(v.shape) if v.dtype == np.uint16 else v.astype(np.float64))
            for k, v in w.items()}


@pytest.mark.parametrize("cfg,seed,bf16", CASES)
def test_numpy_forward_matches_c_forward(cfg, seed, bf16):
    w = _layer(cfg, seed, bf16)
    X = np.random.RandomState(seed + 10).randn(3, cfg["n"], cfg["d"])
    out, _ = oracle.layer_forward_np(cfg, w, X)
    ref = oracle.layer_forward(dict(cfg, layers=1), w, X)
    assert np.allclose(out, ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("cfg,seed,bf16", CASES)
def test_gradients_match_finite_differences(cfg, seed, bf16):
    w = _as_f64(_layer(cfg, seed, bf16))  # float64 parameters, perturbed below
    rng = np.random.RandomState(seed + 20)
    X = rng.randn(3, cfg["n"], cfg["d"])
    dOut = rng.randn(3, cfg["n"], cfg["d"])
    dX, g = oracle.layer_backward(cfg, w, X, dOut)

    def loss(XX, ww):
        return float((oracle.layer_forward_np(cfg, ww, XX)[0] * dOut).sum())

    h = 1e-6
    worst = 0.0
    for flat in rng.choice(X.size, 6, replace=False):
        Xp, Xm = X.copy().reshape(-1), X.copy().reshape(-1)
        Xp[flat] += h
        Xm[flat] -= h
        fd = (loss(Xp.reshape(X.shape), w) - loss(Xm.reshape(X.shape), w)) / (2 * h)
        worst = max(worst, abs(fd - dX.reshape(-1)[flat]) / max(1.0, abs(fd)))
    for name, a in w.items():
        for flat in sorted(set([0, a.size // 2, a.size - 1])):
            ap, am = a.copy().reshape(-1), a.copy().reshape(-1)
            ap[flat] += h
            am[flat] -= h
            fd = (loss(X, dict(w, **{name: ap.reshape(a.shape)})) - loss(X, dict(w, **{name: am.reshape(a.shape)}))) / (2 * h)
            worst = max(worst, abs(fd - g[name].reshape(-1)[flat]) / max(1.0, abs(fd)))
    assert worst < 1e-7, worst


def test_linear_in_the_upstream_gradient():
    cfg, seed, bf16 = CASES[2]
    w = _layer(cfg, seed, bf16)
    rng = np.random.RandomState(7)
    X = rng.randn(2, cfg["n"], cfg["d"])
    d1, d2 = rng.randn(2, cfg["n"], cfg["d"]), rng.randn(2, cfg["n"], cfg["d"])
    a = oracle.layer_backward(cfg, w, X, d1)
    b = oracle.layer_backward(cfg, w, X, d2)
    c = oracle.layer_backward(cfg, w, X, 2.0 * d1 - 3.0 * d2)
    assert np.allclose(c[0], 2.0 * a[0] - 3.0 * b[0], rtol=0, atol=1e-10)
    for key in c[1]:
        assert np.allclose(c[1][key], 2.0 * a[1][key] - 3.0 * b[1][key], rtol=0, atol=1e-10), key


def test_closed_relu_gate_gets_no_weight_gradient():
    cfg = dict(n=4, d=4, k=2, n_f=2, n_l=2, hidden=[5])
    w = _layer(cfg, 4)
    w["b0"] = w["b0"].copy()
    w["W0"] = w["W0"].copy()
    w["W0"][2, :] = 0.0
    w["b0"][2] = -1.0  # unit 2 of the hidden layer is -1 for every input: ReLU closed
    X = np.random.RandomState(5).randn(3, 4, 4)
    dOut = np.random.RandomState(6).randn(3, 4, 4)
    _, g = oracle.layer_backward(cfg, w, X, dOut)
    assert np.all(g["W0"][2, :] == 0.0) and g["b0"][2] == 0.0
    assert np.abs(g["W0"]).sum() > 0.0


def test_layernorm_backward_invariants():
    """The LayerNorm's normalisation is unchanged when a constant is added to its input row,
    and (with eps = 0) when the row is scaled by a positive factor: the exact input gradient
    therefore sums to zero over the row and is orthogonal to the centred row, whatever the
    upstream gradient. A dropped mean term fails the first, a dropped variance term the
    second. Also, against the Jacobian dxhat_i / dx_j = rs (delta_ij - 1/N - xhat_i xhat_j / N)
    built as a matrix."""
    rng = np.random.RandomState(11)
    N = 37
    x = rng.randn(5, N) * 3.0 + 2.0
    g = rng.randn(5, N)
    mu = x.mean(axis=1, keepdims=True)
    for eps in (0.0, 1e-5):
        rs = 1.0 / np.sqrt(((x - mu) ** 2).mean(axis=1, keepdims=True) + eps)
        xh = (x - mu) * rs
        dx = oracle.layernorm_backward(g, xh, rs)
        assert np.allclose(dx.sum(axis=1), 0.0, atol=1e-12)
        if eps == 0.0:
            assert np.allclose((dx * (x - mu)).sum(axis=1), 0.0, atol=1e-11)
        for r in range(5):
            J = rs[r, 0] * (np.eye(N) - 1.0 / N - np.outer(xh[r], xh[r]) / N)
            assert np.allclose(dx[r], J.T @ g[r], rtol=0, atol=1e-12)
