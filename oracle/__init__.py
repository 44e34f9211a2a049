"""fp64 oracle of the Wukong interaction-stack forward -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` import this package. It wraps the plain C reference in
``wk_oracle.c`` (see its header for the equations and their sources on the
Wukong page) and streams a stack one layer at a time, so that a large workload
needs only one layer's weights in host memory.

Parity status: pinned by identities (tests/test_oracle_pins.py); the page prints
no worked example of a whole layer. The chaining of layers (stack_forward, moe_forward)
is pinned by closed-form multi-layer stacks (tests/test_oracle_stack_pins.py). The backward pass (layer_backward, numpy float64,
derived from the forward by the chain rule) is pinned by finite differences of the
forward (tests/test_oracle_backward_pins.py); its ReLU gates are its own float64
decisions (pre-activation > 0), nothing here models a kernel's precision.
"""
import ctypes
import os

import numpy as np

from . import build as _build

_lib = None


class _Config(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("d", ctypes.c_int32), ("k", ctypes.c_int32), ("n_f", ctypes.c_int32),
                ("n_l", ctypes.c_int32), ("mlp_num_linear", ctypes.c_int32),
                ("mlp_dims", ctypes.POINTER(ctypes.c_int32)), ("ln_eps", ctypes.c_double),
                ("dtype", ctypes.c_int32)]


class _Layer(ctypes.Structure):
    _fields_ = [("Y", ctypes.c_void_p), ("W", ctypes.POINTER(ctypes.c_void_p)),
                ("b", ctypes.POINTER(ctypes.c_void_p)), ("fmb_gamma", ctypes.c_void_p),
                ("fmb_beta", ctypes.c_void_p), ("W_L", ctypes.c_void_p), ("out_gamma", ctypes.c_void_p),
                ("out_beta", ctypes.c_void_p)]


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(_build.build())
        vp, i32, i64, dbl = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        L.wko_fm.argtypes = [i32, i32, i32, vp, vp, vp, vp]
        L.wko_layernorm.argtypes = [i64, vp, vp, vp, dbl, vp]
        L.wko_lcb.argtypes = [i32, i32, i32, vp, vp, vp]
        L.wko_layer_forward.argtypes = [ctypes.POINTER(_Config), ctypes.POINTER(_Layer), i64, vp, vp,
                                        ctypes.c_int, ctypes.c_int]
        L.wko_layer_forward.restype = ctypes.c_int
        L.wko_linear.argtypes = [i64, i64, i64, i32, vp, vp, ctypes.c_int, vp, vp]
        L.wko_round_bf16.argtypes = [dbl]
        L.wko_round_bf16.restype = dbl
        _lib = L
    return _lib


def _c64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _ptr(a):
    return None if a is None else a.ctypes.data


def fm(X, Y):
    """F = (X X^T) Y for one example, by pairwise dot products. X [n,d], Y [n,k]."""
    X, Y = _c64(X), _c64(Y)
    n, d = X.shape
    k = Y.shape[1]
    P = np.empty((n, n))
    F = np.empty((n, k))
    lib().wko_fm(n, d, k, _ptr(X), _ptr(Y), _ptr(P), _ptr(F))
    return F


def layernorm(x, gamma=None, beta=None, eps=1e-5):
    x = _c64(x).reshape(-1)
    g = None if gamma is None else _c64(gamma).reshape(-1)
    b = None if beta is None else _c64(beta).reshape(-1)
    y = np.empty_like(x)
    lib().wko_layernorm(x.size, _ptr(x), _ptr(g), _ptr(b), float(eps), _ptr(y))
    return y


def lcb(W_L, X):
    """G = W_L X for one example. W_L [n_l, n], X [n, d]."""
    W_L, X = _c64(W_L), _c64(X)
    n_l, n = W_L.shape
    d = X.shape[1]
    G = np.empty((n_l, d))
    lib().wko_lcb(n, d, n_l, _ptr(W_L), _ptr(X), _ptr(G))
    return G


def linear(x, W, b=None, relu=False):
    """y = act(x W^T + b) on a batch x [n_ex, in]; W float32 [out, in] or uint16 bf16 bits."""
    x = _c64(x)
    W = np.ascontiguousarray(W)
    dt = 1 if W.dtype == np.uint16 else 0
    if dt == 0:
        W = W.astype(np.float32)
    bb = None if b is None else np.ascontiguousarray(b, dtype=np.float32)
    n_ex, i = x.shape
    o = W.shape[0]
    y = np.empty((n_ex, o))
    lib().wko_linear(n_ex, i, o, dt, _ptr(W), _ptr(bb), int(relu), _ptr(x), _ptr(y))
    return y


def round_bf16(v):
    return lib().wko_round_bf16(float(v))


def default_threads():
    return max(1, os.cpu_count() or 1)


def layer_forward(cfg, weights, X, threads=None, diag=0, ln_eps=1e-5):
    """One Wukong layer on host examples X [n_ex, n, d] (float64). ``weights`` is a
    dict with Y, W0..W{m-1}, b0..b{m-1}, fmb_gamma, fmb_beta, W_L, out_gamma,
    out_beta as host arrays (float32, or uint16 bf16 bits for Y / W_j / W_L)."""
    X = _c64(X)
    n_ex = X.shape[0]
    dims = [cfg["n"] * cfg["k"]] + list(cfg["hidden"]) + [cfg["n_f"] * cfg["d"]]
    m = len(dims) - 1
    dims_c = (ctypes.c_int32 * len(dims))(*dims)
    wdt = weights["Y"].dtype
    dtype = 1 if wdt == np.uint16 else 0
    keep = []

    def arr(a, want):
        a = np.ascontiguousarray(a)
        if want == "w":
            assert a.dtype == wdt
        else:
            a = np.ascontiguousarray(a, dtype=np.float32)
        keep.append(a)
        return a.ctypes.data

    c = _Config(cfg["n"], cfg["d"], cfg["k"], cfg["n_f"], cfg["n_l"], m, dims_c, ln_eps, dtype)
    Wp = (ctypes.c_void_p * m)(*[arr(weights["W%d" % j], "w") for j in range(m)])
    bp = (ctypes.c_void_p * m)(*[arr(weights["b%d" % j], "f") if weights.get("b%d" % j) is not None else None
                                  for j in range(m)])
    lay = _Layer(arr(weights["Y"], "w"), Wp, bp, arr(weights["fmb_gamma"], "f"), arr(weights["fmb_beta"], "f"),
                 arr(weights["W_L"], "w"), arr(weights["out_gamma"], "f"), arr(weights["out_beta"], "f"))
    diag = 15 if diag is True else int(diag)
    out = np.empty_like(X)
    rc = lib().wko_layer_forward(ctypes.byref(c), ctypes.byref(lay), n_ex, _ptr(X), _ptr(out),
                                 threads or default_threads(), int(diag))
    if rc:
        raise ValueError("oracle rejected the configuration")
    return out


def stack_forward(cfg, layer_weights, X, threads=None, diag=0):
    """The whole stack, one layer at a time. ``layer_weights(l)`` returns layer l's
    host weights (so a large stack can be generated layer by layer)."""
    h = _c64(X)
    for layer in range(cfg["layers"]):
        h = layer_forward(cfg, layer_weights(layer), h, threads=threads, diag=diag)
    return h


# ------------------------------------------------------------------ Wukong-MoE
#
# Kunlun page (gist.science summary of arXiv 2602.10016), section 2.3, "Wukong Mixture
# of Experts": the global interaction module runs several Wukong modules in parallel as
# the experts of one layer, spreading the layer's computation over them. The page gives
# no formula. Reading taken (the textbook dense mixture of experts): expert e is a whole
# Wukong layer with its own weights; a softmax gate over the experts, computed per
# example from the flattened layer input, weights their outputs:
#   g(X)    = softmax( W_g vec(X) + b_g ),   W_g in R^{E x n d}, vec row-major
#   MoE(X)  = sum_e g_e(X) * WukongLayer_e(X)
# Every expert is evaluated for every example (no top-k routing: the page names none).


def _weight_f64(a):
    a = np.ascontiguousarray(a)
    if a.dtype == np.uint16:
        import synth
        return synth.bf16_bits_to_f64(a).reshape(a.shape)
    return a.astype(np.float64)


def gate_softmax(W_g, b_g, X):
    """g [n_ex, E]: the softmax over experts of W_g vec(X_b) + b_g, in float64.
    W_g [E, n*d] (float32 or bf16 bits), b_g [E] or None, X [n_ex, n, d] float64."""
    X = _c64(X)
    x = X.reshape(X.shape[0], -1)
    logits = x @ _weight_f64(W_g).T
    if b_g is not None:
        logits = logits + np.asarray(b_g, dtype=np.float64)[None, :]
    z = logits - logits.max(axis=1, keepdims=True)
    w = np.exp(z)
    return w / w.sum(axis=1, keepdims=True)


def moe_layer_forward(cfg, expert_weights, gate, X, threads=None, ln_eps=1e-5):
    """One Wukong-MoE layer: expert_weights is a list of E layer-weight dicts (as for
    layer_forward), gate a dict with W_g and b_g; X [n_ex, n, d] float64."""
    X = _c64(X)
    g = gate_softmax(gate["W_g"], gate.get("b_g"), X)
    out = np.zeros_like(X)
    for e, w in enumerate(expert_weights):
        out += g[:, e, None, None] * layer_forward(cfg, w, X, threads=threads, ln_eps=ln_eps)
    return out


def moe_forward(cfg, expert_weights, gate_weights, X, threads=None):
    """The MoE stack, one layer at a time: expert_weights(l, e) and gate_weights(l)
    return host weights of expert e and of the gate of layer l."""
    h = _c64(X)
    for layer in range(cfg["layers"]):
        experts = [expert_weights(layer, e) for e in range(cfg["experts"])]
        h = moe_layer_forward(cfg, experts, gate_weights(layer), h, threads=threads)
    return h


# --------------------------------------------------------------- prediction head
#
# Wukong page, section 2.2, first paragraph: the model first crosses features with the
# stacked Wukong layers and then produces the prediction with an MLP. The page gives
# the head no sizes. Reading taken: the last layer's embeddings are flattened
# row-major, q Linear layers follow with ReLU after all but the last, the last has one
# output (the logit), and the prediction is its logistic sigmoid (a click probability).


def top_mlp_forward(weights, X):
    """(logit [n_ex], p [n_ex]) of the prediction head on X [n_ex, n, d] (float64).
    weights: list of (T_j [out_j, in_j] float32 or bf16 bits, c_j [out_j] float32 or
    None), in_0 = n*d, out_{q-1} = 1."""
    X = _c64(X)
    z = X.reshape(X.shape[0], -1)
    q = len(weights)
    for j, (T, c) in enumerate(weights):
        z = linear(z, T, c, relu=j < q - 1)
    logit = z[:, 0]
    p = 1.0 / (1.0 + np.exp(-logit))
    return logit, p


# ------------------------------------------------------- WHALE attention fusion
#
# WHALE pages (gist.science summaries of arXiv 2607.17017, Korean and French), section 2.1,
# item 3 (attention-based fusion) and section 2.2 (shared K = V; shared-gate SwiGLU with
# W_gate = W_up). The Wukong representation H_w (n rows of d) is the query, the sequence
# representation H_s (L rows of d) is both key and value; the attention output is
# concatenated with H_w, projected by a fusion MLP, and passed through a pre-norm SwiGLU
# FFN whose gate and up projections are one matrix. The pages give no formulas. Readings
# taken (the plainest ones the text supports): one head, no Q/K/V projections (K = V =
# H_s), scaled dot-product scores S = H_w H_s^T / sqrt(d); the fusion MLP is one Linear
# 2d -> d with bias; the FFN is H_f = Z + W_down (SiLU(U) * U), U = W_up LN(Z) (pre-norm:
# LayerNorm over d, then the FFN, then the residual), no FFN biases.


def attention_shared_kv(Hw, Hs):
    """A [n, d] = softmax_rows(Hw Hs^T / sqrt(d)) Hs for one example, in float64."""
    Hw, Hs = _c64(Hw), _c64(Hs)
    d = Hw.shape[1]
    S = (Hw @ Hs.T) / np.sqrt(d)
    S = S - S.max(axis=1, keepdims=True)
    P = np.exp(S)
    P = P / P.sum(axis=1, keepdims=True)
    return P @ Hs


def whale_fusion(Hw, Hs, w, ln_eps=1e-5):
    """H_f [n, d] for one example. w: W_F [d, 2d], b_F [d] (or None), ln_gamma / ln_beta [d],
    W_up [h, d], W_down [d, h] (float32 or bf16 bits)."""
    Hw = _c64(Hw)
    return fusion_ffn(Hw, attention_shared_kv(Hw, Hs), w, ln_eps)


def fusion_ffn(Hw, A, w, ln_eps=1e-5):
    """The part of the fusion after the attention, on rows of H_w [r, d] and A [r, d]:
    Z = [H_w | A] W_F^T + b_F, then Z + W_down(SiLU(U) * U) with U = W_up LN(Z)."""
    Hw, A = _c64(Hw), _c64(A)
    C = np.concatenate([Hw, A], axis=1)
    Z = linear(C, w["W_F"], w.get("b_F"))
    Zn = np.stack([layernorm(z, w["ln_gamma"], w["ln_beta"], ln_eps) for z in Z])
    U = linear(Zn, w["W_up"])
    G = U * U / (1.0 + np.exp(-U))
    return Z + linear(G, w["W_down"])


# ------------------------------------------------------------ backward pass
#
# The gradients of one Wukong layer (the forward of layer_forward: Wukong page, section
# 2.2), derived from that forward by the chain rule; the pages give no backward. Written
# in the plain association of the forward (the FM through P = X X^T, F = P Y), every step
# in float64, vectorised over the examples with einsum. Weight gradients are summed over
# the examples. The ReLU derivative is 1 where the pre-activation is > 0, else 0.


def layer_forward_np(cfg, w, X, ln_eps=1e-5):
    """The layer forward in numpy float64 (the same function as layer_forward's C code),
    returning the output and the intermediates the backward reads."""
    X = _c64(X)
    E, n, d = X.shape
    k, n_f = cfg["k"], cfg["n_f"]
    m = len(cfg["hidden"]) + 1
    Y = _weight_f64(w["Y"])
    Ws = [_weight_f64(w["W%d" % j]) for j in range(m)]
    bs = [np.zeros(Ws[j].shape[0]) if w.get("b%d" % j) is None else _c64(w["b%d" % j]) for j in range(m)]
    g1, b1 = _c64(w["fmb_gamma"]), _c64(w["fmb_beta"])
    W_L = _weight_f64(w["W_L"])
    g2, b2 = _c64(w["out_gamma"]), _c64(w["out_beta"])
    P = np.einsum("eit,ejt->eij", X, X)
    F = np.einsum("eij,jc->eic", P, Y)
    f = F.reshape(E, n * k)
    mu = f.mean(axis=1, keepdims=True)
    rs = 1.0 / np.sqrt(((f - mu) ** 2).mean(axis=1, keepdims=True) + ln_eps)
    fh = (f - mu) * rs
    hs, zs = [fh * g1 + b1], []
    for j in range(m):
        z = hs[-1] @ Ws[j].T + bs[j]
        zs.append(z)
        hs.append(np.maximum(z, 0.0) if j < m - 1 else z)
    G = np.einsum("ri,eit->ert", W_L, X)
    y = np.concatenate([hs[-1].reshape(E, n_f, d), G], axis=1) + X
    mu2 = y.mean(axis=2, keepdims=True)
    rs2 = 1.0 / np.sqrt(((y - mu2) ** 2).mean(axis=2, keepdims=True) + ln_eps)
    yh = (y - mu2) * rs2
    out = yh * g2 + b2
    return out, dict(X=X, P=P, fh=fh, rs=rs, hs=hs, zs=zs, yh=yh, rs2=rs2, Y=Y, Ws=Ws, g1=g1, W_L=W_L, g2=g2)


def layernorm_backward(dxh, xh, rs):
    """d/dx of the normalisation xh = (x - mean) * rs over the last axis, given d/dxh."""
    return rs * (dxh - dxh.mean(axis=-1, keepdims=True) - xh * (dxh * xh).mean(axis=-1, keepdims=True))


def layer_backward(cfg, w, X, dOut, ln_eps=1e-5):
    """(dX [E, n, d], grads) of one layer at X for the upstream gradient dOut = dL/d(output).
    grads: Y, W0.., b0.., fmb_gamma, fmb_beta, W_L, out_gamma, out_beta (float64, summed
    over the E examples). Weights as for layer_forward (float32 or bf16 bits). The ReLU
    derivative is 1 where the float64 pre-activation is > 0, else 0."""
    _, c = layer_forward_np(cfg, w, X, ln_eps)
    dOut = _c64(dOut)
    E, n, d = c["X"].shape
    k, n_f = cfg["k"], cfg["n_f"]
    m = len(c["Ws"])
    g = {}
    # output LayerNorm per embedding row, residual, concat
    g["out_gamma"] = (dOut * c["yh"]).sum(axis=(0, 1))
    g["out_beta"] = dOut.sum(axis=(0, 1))
    dy = layernorm_backward(dOut * c["g2"], c["yh"], c["rs2"])
    dX = dy.copy()
    # LCB: G = W_L X
    dG = dy[:, n_f:, :]
    g["W_L"] = np.einsum("ert,eit->ri", dG, c["X"])
    dX += np.einsum("ri,ert->eit", c["W_L"], dG)
    # FMB MLP, last Linear first
    dh = dy[:, :n_f, :].reshape(E, n_f * d)
    for j in range(m - 1, -1, -1):
        if j < m - 1:
            dz = dh * (c["zs"][j] > 0.0)
        else:
            dz = dh
        g["W%d" % j] = dz.T @ c["hs"][j]
        g["b%d" % j] = dz.sum(axis=0)
        dh = dz @ c["Ws"][j]
    # FMB LayerNorm over the flattened n*k values
    g["fmb_gamma"] = (dh * c["fh"]).sum(axis=0)
    g["fmb_beta"] = dh.sum(axis=0)
    dF = layernorm_backward(dh * c["g1"], c["fh"], c["rs"]).reshape(E, n, k)
    # FM: F = P Y, P = X X^T (symmetric)
    g["Y"] = np.einsum("eij,ejc->ic", c["P"], dF)
    dP = np.einsum("eic,jc->eij", dF, c["Y"])
    dX += np.einsum("eij,ejt->eit", dP + dP.transpose(0, 2, 1), c["X"])
    return dX, g
