"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
hand-worked fixtures (tests/golden), exact rational arithmetic, the other
association of the FM product, closed forms, and special cases that reduce to a
library routine (numpy matmul, torch LayerNorm). Each case is chosen so that a
plausible slip in the oracle (a dropped term, a transposed operand, a wrong
variance, a swapped concat order, a ReLU on the last Linear, a wrong flatten
order) fails at least one of them.

Method source: the Wukong page (xdnf.cn repost of "Wukong: Towards a Scaling
Law for Large-Scale Recommendation"), section 2.2 (Wukong layer, FMB, LCB) and
section 2.3 (knobs).
"""
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_cases(name):
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "case":
            cur = {}
            cases.append(cur)
            continue
        if len(parts) >= 2 and not parts[0][0].isdigit() and not parts[0][0] == "-":
            cur[parts[0]] = [float(v) for v in parts[1:]]
        else:
            cur["dims"] = [int(v) for v in parts]
    return cases


# ---------------------------------------------------------------- FM ------

def test_fm_golden_hand_worked():
    for case in _read_cases("fm_tiny.txt"):
        _, n, d, k = case["dims"]
        X = np.array(case["X"]).reshape(n, d)
        Y = np.array(case["Y"]).reshape(n, k)
        F = oracle.fm(X, Y)
        assert np.array_equal(F, np.array(case["F"]).reshape(n, k))


def test_fm_exact_rational_reassociation():
    """(X X^T) Y from the oracle equals X (X^T Y) computed in exact rationals."""
    rng = np.random.RandomState(3)
    for n, d, k in [(3, 2, 1), (4, 3, 2), (2, 4, 3), (4, 4, 4)]:
        X = rng.randint(-5, 6, size=(n, d))
        Y = rng.randint(-5, 6, size=(n, k))
        XtY = [[sum(Fraction(int(X[i][t])) * int(Y[i][c]) for i in range(n)) for c in range(k)] for t in range(d)]
        ref = [[sum(Fraction(int(X[i][t])) * XtY[t][c] for t in range(d)) for c in range(k)] for i in range(n)]
        F = oracle.fm(X.astype(float), Y.astype(float))
        for i in range(n):
            for c in range(k):
                assert Fraction(F[i][c]) == ref[i][c]


def test_fm_reassociation_fp64_random():
    """The optimised association X (X^T Y) (numpy matmul) agrees to rounding, n != d != k."""
    rng = np.random.RandomState(0)
    for n, d, k in [(16, 16, 4), (37, 11, 5), (64, 128, 16)]:
        X = rng.randn(n, d)
        Y = rng.randn(n, k)
        F = oracle.fm(X, Y)
        ref = X @ (X.T @ Y)
        assert np.max(np.abs(F - ref)) <= 1e-12 * (1 + np.max(np.abs(ref)))


def test_fm_orthogonal_rows_closed_form():
    """Orthogonal rows make X X^T diagonal: F[i] = |x_i|^2 y_i."""
    rng = np.random.RandomState(1)
    n, d, k = 5, 8, 3
    Q, _ = np.linalg.qr(rng.randn(d, d))
    scales = rng.uniform(0.5, 2.0, size=n)
    X = Q[:n] * scales[:, None]
    Y = rng.randn(n, k)
    F = oracle.fm(X, Y)
    assert np.allclose(F, (scales ** 2)[:, None] * Y, rtol=1e-12, atol=1e-12)


def test_fm_homogeneity_and_linearity():
    rng = np.random.RandomState(2)
    X, Y1, Y2 = rng.randn(9, 6), rng.randn(9, 4), rng.randn(9, 4)
    assert np.allclose(oracle.fm(2.5 * X, Y1), 6.25 * oracle.fm(X, Y1), rtol=1e-12)
    assert np.allclose(oracle.fm(X, Y1 + Y2), oracle.fm(X, Y1) + oracle.fm(X, Y2), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- LCB -----

def test_lcb_identity_returns_x():
    rng = np.random.RandomState(4)
    X = rng.randn(7, 5)
    assert np.array_equal(oracle.lcb(np.eye(7), X), X)


def test_lcb_permutation_and_library_matmul():
    rng = np.random.RandomState(5)
    X = rng.randn(6, 3)
    P = np.eye(6)[[3, 0, 5]]  # n_l = 3 rows picking features 3, 0, 5
    assert np.array_equal(oracle.lcb(P, X), X[[3, 0, 5]])
    W = rng.randn(4, 6)
    assert np.allclose(oracle.lcb(W, X), W @ X, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------- LN ------

def test_layernorm_golden_hand_worked():
    for case in _read_cases("layernorm_tiny.txt"):
        y = oracle.layernorm(case["x"], case["gamma"], case["beta"], eps=case["eps"][0])
        assert np.allclose(y, case["y"], rtol=0, atol=1e-14)


def test_layernorm_moments_closed_form():
    """gamma=1, beta=0: mean 0 and variance var/(var+eps) exactly (up to rounding)."""
    rng = np.random.RandomState(6)
    for scale in (1e-3, 1.0, 30.0):
        x = rng.randn(160) * scale + 0.7
        eps = 1e-5
        y = oracle.layernorm(x, eps=eps)
        var = np.var(x)
        assert abs(np.mean(y)) <= 1e-12
        assert abs(np.var(y) - var / (var + eps)) <= 1e-12


def test_layernorm_matches_torch_library():
    rng = np.random.RandomState(7)
    x = rng.randn(3, 48) * 2.0
    g, b = rng.randn(48), rng.randn(48)
    for r in range(3):
        ref = torch.nn.functional.layer_norm(torch.tensor(x[r]), (48,), torch.tensor(g), torch.tensor(b), 1e-5)
        assert np.allclose(oracle.layernorm(x[r], g, b), ref.numpy(), rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- MLP -----

def test_linear_identity_and_relu():
    rng = np.random.RandomState(8)
    x = rng.randn(4, 6)
    eye = np.eye(6, dtype=np.float32)
    assert np.array_equal(oracle.linear(x, eye), x)
    assert np.array_equal(oracle.linear(x, eye, relu=True), np.maximum(x, 0.0))
    W = rng.randn(5, 6).astype(np.float32)
    b = rng.randn(5).astype(np.float32)
    assert np.allclose(oracle.linear(x, W, b), x @ W.astype(np.float64).T + b, rtol=1e-13, atol=1e-13)


def test_linear_bf16_weights_upcast_exactly():
    w = np.array([[0x3F80, 0xBF00], [0x4040, 0x0000]], dtype=np.uint16)  # [[1, -0.5], [3, 0]]
    y = oracle.linear(np.array([[2.0, 4.0]]), w)
    assert np.array_equal(y, np.array([[0.0, 6.0]]))


# ---------------------------------------------------------------- layer ---

def _layer_weights(n, d, k, n_f, n_l, hidden, zero=True, rng=None):
    dims = [n * k] + list(hidden) + [n_f * d]
    w = {}
    for j in range(len(dims) - 1):
        w["W%d" % j] = np.zeros((dims[j + 1], dims[j]), np.float32)
        w["b%d" % j] = np.zeros(dims[j + 1], np.float32)
    w["Y"] = np.zeros((n, k), np.float32)
    w["W_L"] = np.zeros((n_l, n), np.float32)
    w["fmb_gamma"] = np.ones(n * k, np.float32)
    w["fmb_beta"] = np.zeros(n * k, np.float32)
    w["out_gamma"] = np.ones(d, np.float32)
    w["out_beta"] = np.zeros(d, np.float32)
    return w


def _cfg(n, d, k, n_f, n_l, hidden):
    return dict(n=n, d=d, k=k, n_f=n_f, n_l=n_l, hidden=list(hidden), layers=1)


def _torch_ln_rows(x, g=None, b=None, eps=1e-5):
    t = torch.tensor(x)
    G = None if g is None else torch.tensor(np.asarray(g, np.float64))
    B = None if b is None else torch.tensor(np.asarray(b, np.float64))
    return torch.nn.functional.layer_norm(t, (x.shape[-1],), G, B, eps).numpy()


def test_layer_all_zero_weights_reduces_to_layernorm_of_x():
    """Y, W_j, b_j, W_L all zero: the FMB LayerNorm sees a zero vector (output 0),
    the MLP and LCB give 0, so the layer is LN_d(X) row by row."""
    n, d, k, n_f, n_l = 8, 6, 3, 5, 3
    cfg = _cfg(n, d, k, n_f, n_l, [7])
    w = _layer_weights(n, d, k, n_f, n_l, [7])
    X = np.random.RandomState(9).randn(3, n, d)
    out = oracle.layer_forward(cfg, w, X)
    assert np.allclose(out, _torch_ln_rows(X), rtol=1e-12, atol=1e-12)


def test_layer_concat_order_and_residual():
    """Last MLP bias c (all weights zero) makes every FMB row the constant c; W_L
    selects features 0..n_l-1. Rows 0..n_f-1 must be LN(c + x_r) and rows
    n_f + r must be LN(x_r + x_{n_f + r})."""
    n, d, k, n_f, n_l = 7, 4, 2, 4, 3
    cfg = _cfg(n, d, k, n_f, n_l, [5])
    w = _layer_weights(n, d, k, n_f, n_l, [5])
    c = np.linspace(-1.5, 2.0, n_f * d).astype(np.float32)
    w["b1"] = c
    w["W_L"] = np.eye(n, dtype=np.float32)[:n_l]
    X = np.random.RandomState(10).randn(2, n, d)
    out = oracle.layer_forward(cfg, w, X)
    cm = c.astype(np.float64).reshape(n_f, d)
    for e in range(2):
        assert np.allclose(out[e, :n_f], _torch_ln_rows(cm + X[e, :n_f]), rtol=1e-12, atol=1e-12)
        assert np.allclose(out[e, n_f:], _torch_ln_rows(X[e, :n_l] + X[e, n_f:]), rtol=1e-12, atol=1e-12)


def test_layer_fmb_flatten_order_with_identity_mlp():
    """With n*k == n_f*d and a single identity Linear, the FMB block is
    reshape(LN(flatten(F)) * gamma + beta) with per-position gamma/beta; F comes
    from the other association X (X^T Y). A wrong flatten order, a ReLU on the last
    Linear or a transposed FM operand changes the result."""
    n, d, k, n_f, n_l = 6, 3, 2, 4, 2
    assert n * k == n_f * d
    rng = np.random.RandomState(11)
    cfg = _cfg(n, d, k, n_f, n_l, [])
    w = _layer_weights(n, d, k, n_f, n_l, [])
    w["W0"] = np.eye(n * k, dtype=np.float32)
    w["Y"] = rng.randn(n, k).astype(np.float32)
    w["fmb_gamma"] = rng.uniform(0.5, 1.5, n * k).astype(np.float32)
    w["fmb_beta"] = rng.randn(n * k).astype(np.float32)
    X = rng.randn(2, n, d)
    out = oracle.layer_forward(cfg, w, X)
    Y = w["Y"].astype(np.float64)
    for e in range(2):
        F = X[e] @ (X[e].T @ Y)
        a0 = _torch_ln_rows(F.reshape(-1), w["fmb_gamma"], w["fmb_beta"])
        fmb = a0.reshape(n_f, d)  # negative entries must survive: no ReLU after the last Linear
        assert (fmb < 0).any()
        cat = np.concatenate([fmb, np.zeros((n_l, d))]) + X[e]
        assert np.allclose(out[e], _torch_ln_rows(cat), rtol=1e-11, atol=1e-11)


def test_layer_hidden_relu_is_applied():
    """A hidden Linear of -I followed by an identity output: ReLU(-a0) survives only
    where a0 < 0, so the FMB rows are max(-a0, 0)."""
    n, d, k, n_f, n_l = 4, 2, 1, 2, 2
    rng = np.random.RandomState(12)
    cfg = _cfg(n, d, k, n_f, n_l, [n * k])
    w = _layer_weights(n, d, k, n_f, n_l, [n * k])
    w["W0"] = -np.eye(n * k, dtype=np.float32)
    w["W1"] = np.eye(n * k, dtype=np.float32)
    w["Y"] = rng.randn(n, k).astype(np.float32)
    X = rng.randn(1, n, d)
    out = oracle.layer_forward(cfg, w, X)
    F = X[0] @ (X[0].T @ w["Y"].astype(np.float64))
    a0 = _torch_ln_rows(F.reshape(-1))
    fmb = np.maximum(-a0, 0.0).reshape(n_f, d)
    cat = np.concatenate([fmb, np.zeros((n_l, d))]) + X[0]
    assert np.allclose(out[0], _torch_ln_rows(cat), rtol=1e-11, atol=1e-11)


def test_oracle_rejects_mismatched_residual():
    cfg = _cfg(8, 4, 2, 5, 4, [3])  # n_f + n_l != n
    w = _layer_weights(8, 4, 2, 5, 4, [3])
    with pytest.raises(ValueError):
        oracle.layer_forward(cfg, w, np.zeros((1, 8, 4)))


def test_diag_rounding_matches_torch_bf16():
    rng = np.random.RandomState(13)
    vals = rng.randn(2000).astype(np.float32).astype(np.float64) * 3
    ref = torch.tensor(vals, dtype=torch.float32).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.round_bf16(v) for v in vals])
    assert np.array_equal(got, ref)
