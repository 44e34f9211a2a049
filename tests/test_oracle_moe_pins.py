"""Pins of the Wukong mixture-of-experts oracle (Kunlun page, section 2.3, "Wukong
Mixture of Experts": several Wukong modules run in parallel as the experts of one
layer). Reading: MoE(X) = sum_e g_e(X) WukongLayer_e(X), g = softmax(W_g vec(X) + b_g).

Each pin is a fact that does not come from the oracle: a hand-worked gate
(tests/golden/moe_gate_tiny.txt), softmax closed forms (equal logits give 1/E; a
dominant logit selects one expert; a shift of every logit changes nothing), the
convex-combination identity (identical experts give that expert), and the one-expert
case, which reduces to the plain Wukong layer that tests/test_oracle_pins.py pins.
A slip in the gate (a transposed W_g, a column-major vec, a missing bias, a missing
normalisation) or in the mixing (a dropped expert, unnormalised weights) fails one.
"""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

CFG = dict(layers=1, experts=3, n=8, d=8, k=4, n_f=4, n_l=4, hidden=[16])


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
        elif parts[0][0].isdigit():
            cur["dims"] = [int(v) for v in parts]
        else:
            cur[parts[0]] = [float(v) for v in parts[1:]]
    return cases


def _layer(rng, cfg):
    n, d, k, n_f, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_f"], cfg["n_l"]
    dims = [n * k] + cfg["hidden"] + [n_f * d]
    w = {"Y": (rng.randn(n, k) / np.sqrt(n)).astype(np.float32),
         "W_L": (rng.randn(n_l, n) / np.sqrt(n)).astype(np.float32),
         "fmb_gamma": (1 + 0.1 * rng.randn(n * k)).astype(np.float32),
         "fmb_beta": (0.1 * rng.randn(n * k)).astype(np.float32),
         "out_gamma": (1 + 0.1 * rng.randn(d)).astype(np.float32),
         "out_beta": (0.1 * rng.randn(d)).astype(np.float32)}
    for j in range(len(dims) - 1):
        w["W%d" % j] = (rng.randn(dims[j + 1], dims[j]) / np.sqrt(dims[j])).astype(np.float32)
        w["b%d" % j] = (0.1 * rng.randn(dims[j + 1])).astype(np.float32)
    return w


def _setup(seed=0, E=3):
    rng = np.random.RandomState(seed)
    cfg = dict(CFG, experts=E)
    experts = [_layer(rng, cfg) for _ in range(E)]
    nd = cfg["n"] * cfg["d"]
    gate = {"W_g": (rng.randn(E, nd) / np.sqrt(nd)).astype(np.float32),
            "b_g": rng.randn(E).astype(np.float32)}
    X = rng.randn(5, cfg["n"], cfg["d"])
    return cfg, experts, gate, X


def test_gate_hand_worked():
    for case in _read_cases("moe_gate_tiny.txt"):
        _, E, n, d = case["dims"]
        X = np.array(case["X"]).reshape(1, n, d)
        W = np.array(case["W"], dtype=np.float32).reshape(E, n * d)
        g = oracle.gate_softmax(W, np.array(case["b"], dtype=np.float32), X)
        assert np.allclose(g[0], case["g"], rtol=0, atol=1e-7), (g, case["g"])


def test_gate_rows_are_distributions_and_flatten_is_row_major():
    cfg, _, gate, X = _setup(1)
    g = oracle.gate_softmax(gate["W_g"], gate["b_g"], X)
    assert np.all(g > 0) and np.allclose(g.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    # a one-hot gate row at flat index i*d + t reads X[i, t]: with two experts, one
    # reading X[2, 5] and one reading nothing, g_0 = sigmoid(X[2, 5])
    n, d = cfg["n"], cfg["d"]
    W = np.zeros((2, n * d), dtype=np.float32)
    W[0, 2 * d + 5] = 1.0
    g = oracle.gate_softmax(W, None, X)
    assert np.allclose(g[:, 0], 1.0 / (1.0 + np.exp(-X[:, 2, 5])), rtol=0, atol=1e-15)


def test_one_expert_is_the_plain_layer():
    cfg, experts, gate, X = _setup(2, E=1)
    got = oracle.moe_layer_forward(cfg, experts, gate, X)
    assert np.array_equal(got, oracle.layer_forward(cfg, experts[0], X))


def test_identical_experts_give_that_expert():
    cfg, experts, gate, X = _setup(3)
    same = [experts[0]] * cfg["experts"]
    got = oracle.moe_layer_forward(cfg, same, gate, X)
    ref = oracle.layer_forward(cfg, experts[0], X)
    assert np.allclose(got, ref, rtol=0, atol=1e-13)


def test_equal_logits_average_the_experts():
    cfg, experts, gate, X = _setup(4)
    flat = {"W_g": np.zeros_like(gate["W_g"]), "b_g": np.full(cfg["experts"], 0.7, dtype=np.float32)}
    got = oracle.moe_layer_forward(cfg, experts, flat, X)
    each = [oracle.layer_forward(cfg, w, X) for w in experts]
    assert np.allclose(got, sum(each) / cfg["experts"], rtol=0, atol=1e-13)


def test_dominant_logit_selects_one_expert():
    cfg, experts, gate, X = _setup(5)
    for j in range(cfg["experts"]):
        b = np.zeros(cfg["experts"], dtype=np.float32)
        b[j] = 1000.0
        got = oracle.moe_layer_forward(cfg, experts, {"W_g": gate["W_g"], "b_g": b}, X)
        assert np.allclose(got, oracle.layer_forward(cfg, experts[j], X), rtol=0, atol=1e-12)


def test_shifting_every_logit_changes_nothing():
    cfg, experts, gate, X = _setup(6)
    a = oracle.moe_layer_forward(cfg, experts, gate, X)
    # the shift is exact in float64 (the gate's arithmetic type); a float32 sum would
    # round the biases themselves
    shifted = {"W_g": gate["W_g"], "b_g": gate["b_g"].astype(np.float64) + 3.0}
    b = oracle.moe_layer_forward(cfg, experts, shifted, X)
    assert np.allclose(a, b, rtol=0, atol=1e-12)
    # and the gate does depend on the input: two examples get different weights
    g = oracle.gate_softmax(gate["W_g"], gate["b_g"], X)
    assert np.max(np.abs(g[0] - g[1])) > 1e-3


def test_bf16_gate_weights_upcast_exactly():
    import synth
    cfg, _, gate, X = _setup(7)
    bits = np.array([synth.f64_to_bf16_bits_scalar(float(v)) for v in gate["W_g"].reshape(-1)],
                    dtype=np.uint16).reshape(gate["W_g"].shape)
    as_f32 = synth.bf16_bits_to_f64(bits).reshape(bits.shape).astype(np.float32)
    assert np.array_equal(oracle.gate_softmax(bits, gate["b_g"], X), oracle.gate_softmax(as_f32, gate["b_g"], X))
