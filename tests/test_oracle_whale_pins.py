"""Pins of the WHALE attention-fusion oracle (WHALE pages, section 2.1 item 3 and section
2.2). Reading: one head, K = V = H_s, S = H_w H_s^T / sqrt(d), A = softmax_rows(S) H_s; the
fusion MLP is one Linear 2d -> d; H_f = Z + W_down(SiLU(U) * U) with U = W_up LN(Z).

Facts that do not come from the oracle: hand-worked attention (tests/golden/
whale_attention_tiny.txt), one key (A is that key), identical keys, permutation invariance
over keys, a dominant score, the fusion and FFN special cases (a selecting W_F with a zero
FFN returns H_w; the attention half of W_F alone returns A; a one-hot W_down reads one
gated unit, compared with SiLU(u) * u written from the definition of the logistic
function). A transposed score matrix, a missing 1/sqrt(d), K and V confused with Q, a
swapped concat order, a post-norm FFN or an ungated SwiGLU fails one of them.
"""
import os

import numpy as np

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _cases():
    cases, cur = [], None
    for line in open(os.path.join(GOLDEN, "whale_attention_tiny.txt")):
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


def test_attention_hand_worked():
    for c in _cases():
        _, n, L, d = c["dims"]
        A = oracle.attention_shared_kv(np.array(c["Hw"]).reshape(n, d), np.array(c["Hs"]).reshape(L, d))
        assert np.allclose(A.reshape(-1), c["A"], rtol=0, atol=1e-12)


def test_attention_closed_forms():
    rng = np.random.RandomState(0)
    Hw = rng.randn(5, 8)
    k = rng.randn(1, 8)
    assert np.allclose(oracle.attention_shared_kv(Hw, k), np.repeat(k, 5, axis=0), rtol=0, atol=1e-14)
    same = np.repeat(k, 7, axis=0)
    assert np.allclose(oracle.attention_shared_kv(Hw, same), np.repeat(k, 5, axis=0), rtol=0, atol=1e-14)
    Hs = rng.randn(9, 8)
    perm = rng.permutation(9)
    assert np.allclose(oracle.attention_shared_kv(Hw, Hs), oracle.attention_shared_kv(Hw, Hs[perm]), rtol=0,
                       atol=1e-13)
    # a query aligned with one key far more than with the others attends to that key
    Hs2 = np.eye(8)[:4] * 1.0
    q = np.zeros((1, 8))
    q[0, 2] = 200.0
    assert np.allclose(oracle.attention_shared_kv(q, Hs2), Hs2[2:3], rtol=0, atol=1e-12)


def _weights(rng, d, h):
    return {"W_F": (rng.randn(d, 2 * d) / np.sqrt(2 * d)).astype(np.float32),
            "b_F": (0.1 * rng.randn(d)).astype(np.float32),
            "ln_gamma": (1 + 0.1 * rng.randn(d)).astype(np.float32),
            "ln_beta": (0.1 * rng.randn(d)).astype(np.float32),
            "W_up": (rng.randn(h, d) / np.sqrt(d)).astype(np.float32),
            "W_down": (rng.randn(d, h) / np.sqrt(h)).astype(np.float32)}


def test_fusion_special_cases():
    rng = np.random.RandomState(1)
    n, L, d, h = 4, 6, 8, 16
    Hw, Hs = rng.randn(n, d), rng.randn(L, d)
    w = _weights(rng, d, h)
    # W_F = [I | 0], no bias, W_down = 0: H_f = H_w
    w0 = dict(w, W_F=np.concatenate([np.eye(d), np.zeros((d, d))], axis=1).astype(np.float32), b_F=None,
              W_down=np.zeros((d, h), dtype=np.float32))
    assert np.allclose(oracle.whale_fusion(Hw, Hs, w0), Hw, rtol=0, atol=1e-14)
    # W_F = [0 | I]: the fused representation starts from the attention output
    w1 = dict(w0, W_F=np.concatenate([np.zeros((d, d)), np.eye(d)], axis=1).astype(np.float32))
    assert np.allclose(oracle.whale_fusion(Hw, Hs, w1), oracle.attention_shared_kv(Hw, Hs), rtol=0, atol=1e-14)


def test_ffn_is_pre_norm_shared_gate_swiglu():
    rng = np.random.RandomState(2)
    n, L, d, h = 3, 5, 8, 16
    Hw, Hs = rng.randn(n, d), rng.randn(L, d)
    w = _weights(rng, d, h)
    # a one-hot W_down row picks gated unit 3 into output column 5
    Wd = np.zeros((d, h), dtype=np.float32)
    Wd[5, 3] = 1.0
    got = oracle.whale_fusion(Hw, Hs, dict(w, W_down=Wd))
    wz = dict(w, W_down=np.zeros((d, h), dtype=np.float32))
    Z = oracle.whale_fusion(Hw, Hs, wz)                       # the FFN input (residual only)
    Zn = (Z - Z.mean(axis=1, keepdims=True)) / np.sqrt(Z.var(axis=1, keepdims=True) + 1e-5)
    Zn = Zn * w["ln_gamma"].astype(np.float64) + w["ln_beta"].astype(np.float64)
    u = Zn @ w["W_up"].astype(np.float64)[3]
    gated = u * (u * (1.0 / (1.0 + np.exp(-u))))            # SiLU(u) * u
    expect = Z.copy()
    expect[:, 5] += gated
    assert np.allclose(got, expect, rtol=0, atol=1e-12)
