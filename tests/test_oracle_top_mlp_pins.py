"""Pins of the prediction-head oracle (Wukong page, section 2.2: after the Wukong
layers, an MLP produces the prediction). Reading: flatten row-major, Linear layers
with ReLU after all but the last, one output logit, logistic sigmoid.

Pins that do not come from the oracle: hand-worked heads (tests/golden/top_mlp_tiny.txt:
a ReLU that clips, biases, a row-major flatten with n > 1), a one-hot single Linear
that reads one input element (flatten order), the sigmoid's closed forms, and the
logit's linearity in the last Linear. A transposed weight, a column-major flatten, a
ReLU on the output, a dropped bias or a wrong sigmoid fails one of them.
"""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "top_mlp_tiny.txt")):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        parts = line.split()
        if parts[0] == "case":
            cur = {}
            cases.append(cur)
        elif parts[0][0].isdigit():
            cur["dims"] = [int(v) for v in parts]
        else:
            cur[parts[0]] = [float(v) for v in parts[1:]]
    return cases


def _weights(case):
    ws, j = [], 0
    while "T%d" % j in case:
        t = case["T%d" % j]
        o, i = int(t[0]), int(t[1])
        ws.append((np.array(t[2:], dtype=np.float32).reshape(o, i), np.array(case["c%d" % j], dtype=np.float32)))
        j += 1
    return ws


def test_hand_worked_heads():
    for case in _cases():
        _, n, d = case["dims"]
        X = np.array(case["X"]).reshape(1, n, d)
        logit, p = oracle.top_mlp_forward(_weights(case), X)
        assert np.allclose(logit, case["logit"], rtol=0, atol=1e-12)
        assert np.allclose(p, case["p"], rtol=0, atol=1e-12)


def test_one_hot_linear_reads_one_element_row_major():
    rng = np.random.RandomState(0)
    n, d = 5, 8
    X = rng.randn(7, n, d)
    for i, t in [(0, 0), (2, 5), (4, 7)]:
        T = np.zeros((1, n * d), dtype=np.float32)
        T[0, i * d + t] = 1.0
        logit, _ = oracle.top_mlp_forward([(T, np.array([0.25], dtype=np.float32))], X)
        assert np.array_equal(logit, X[:, i, t] + 0.25)


def test_sigmoid_closed_forms():
    X = np.array([0.0, 3.0, -3.0, 40.0]).reshape(4, 1, 1)
    _, p = oracle.top_mlp_forward([(np.ones((1, 1), dtype=np.float32), None)], X)
    assert p[0] == 0.5
    assert np.isclose(p[1] + p[2], 1.0, rtol=0, atol=1e-15)
    assert np.isclose(p[1], 1.0 / (1.0 + np.exp(-3.0)), rtol=0, atol=1e-15)
    assert 1.0 - p[3] < 1e-16


def test_logit_is_linear_in_the_last_layer_and_hidden_relu_applies():
    rng = np.random.RandomState(1)
    n, d, h = 3, 8, 16
    X = rng.randn(6, n, d)
    T0 = (rng.randn(h, n * d) / np.sqrt(n * d)).astype(np.float32)
    c0 = rng.randn(h).astype(np.float32)
    # quarter-integers, so that a + b is exact in float32
    a = (rng.randint(-8, 9, size=(1, h)) / 4.0).astype(np.float32)
    b = (rng.randint(-8, 9, size=(1, h)) / 4.0).astype(np.float32)
    la, _ = oracle.top_mlp_forward([(T0, c0), (a, None)], X)
    lb, _ = oracle.top_mlp_forward([(T0, c0), (b, None)], X)
    lab, _ = oracle.top_mlp_forward([(T0, c0), (a + b, None)], X)
    assert np.allclose(lab, la + lb, rtol=0, atol=1e-12)
    # the hidden activation is max(0, .): with the last Linear all ones the logit is the
    # sum of the positive parts of the hidden pre-activations
    pre = X.reshape(6, -1) @ T0.astype(np.float64).T + c0
    ones, _ = oracle.top_mlp_forward([(T0, c0), (np.ones((1, h), dtype=np.float32), None)], X)
    assert np.allclose(ones, np.maximum(pre, 0).sum(axis=1), rtol=0, atol=1e-12)
