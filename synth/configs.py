"""The five synthetic workloads of the Wukong stack forward and their input recipes.

Shapes follow the Wukong page (xdnf.cn repost of "Wukong: Towards a Scaling Law
for Large-Scale Recommendation", section 2.3, the scaling knobs l, n_F, n_L, k
and the FMB MLP) with sizes chosen to match its workloads: embedding dim 160
and 720 features (section 3.2.1). Inputs are synthetic (no dataset):

* X ~ N(0, 1); the wide/narrow workload scales the rows of feature i by
  s_i ~ LogUniform(0.1, 10), one draw per feature shared by all examples.
* Y, W_j, W_L ~ N(0, 1/fan_in) with fan_in = n for Y and W_L and h_j for W_j.
* Biases are 0. LayerNorm gamma = 1, beta = 0, except the 2-layer bf16
  workload, whose LayerNorm affine parameters (both gamma and beta of both
  LayerNorms) are 1 + N(0, 0.02^2).
* Seed 0 for every workload; each tensor has its own stream id (below).

"MLP of m layers of width W" means m Linear layers h_0 = n*k -> W -> ... -> W ->
h_m = n_F*d (m-1 hidden widths, ReLU after each hidden Linear, none after the
last one).
"""
import math

import numpy as np

from . import BF16, F32, bf16_bits_to_f64, fill_normal_host, fill_x_logscaled_host

SEED = 0

# stream ids
TID_X = 1
TID_X_SCALE = 2


def layer_tid(layer, what, j=0):
    base = 1000 * (layer + 1)
    return base + {"Y": 1, "W": 10 + j, "b": 40 + j, "fmb_gamma": 70, "fmb_beta": 71, "W_L": 80,
                   "out_gamma": 90, "out_beta": 91}[what]


CONFIGS = {
    # name: (layers, batch, n, d, k, n_f, n_l, hidden widths, dtype, ln affine, x distribution)
    "c1_fp32": dict(layers=1, batch=64, n=16, d=16, k=4, n_f=8, n_l=8, hidden=[64], dtype="f32",
                    ln_affine="unit", x_dist="normal",
                    about="1-layer fp32, B=64, n=16, d=16, k=4, MLP 64->64->128"),
    "c2_bf16": dict(layers=2, batch=4096, n=64, d=128, k=16, n_f=32, n_l=32, hidden=[1024], dtype="bf16",
                    ln_affine="1+N(0,0.02)", x_dist="normal",
                    about="2-layer bf16, B=4096, n=64, d=128, k=16, MLP 1024->1024->4096"),
    "c3_bf16": dict(layers=4, batch=16384, n=256, d=160, k=32, n_f=128, n_l=128, hidden=[4096, 4096],
                    dtype="bf16", ln_affine="unit", x_dist="normal",
                    about="4-layer bf16 (~1.14 GFLOP/example), B=16384, n=256, d=160, k=32"),
    "c4_bf16": dict(layers=8, batch=4096, n=512, d=160, k=64, n_f=256, n_l=256, hidden=[16384, 16384],
                    dtype="bf16", ln_affine="unit", x_dist="normal",
                    about="8-layer bf16 (~24.1 GFLOP/example), B=4096, n=512, d=160, k=64"),
    "c5_bf16": dict(layers=2, batch=32768, n=720, d=32, k=24, n_f=360, n_l=360, hidden=[2048], dtype="bf16",
                    ln_affine="unit", x_dist="logscaled",
                    about="2-layer wide-feature narrow-dim bf16, B=32768, n=720, d=32, k=24"),
}


def mlp_dims(cfg):
    """[h_0, ..., h_m]: h_0 = n*k, the hidden widths, h_m = n_F*d."""
    return [cfg["n"] * cfg["k"]] + list(cfg["hidden"]) + [cfg["n_f"] * cfg["d"]]


def flops_per_example(cfg):
    """Matmul FLOPs (2 per multiply-add) of one example through the stack:
    L * (4 n d k + 2 n_L n d + 2 sum_j h_j h_{j+1})."""
    n, d, k, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_l"]
    h = mlp_dims(cfg)
    per_layer = 4 * n * d * k + 2 * n_l * n * d + 2 * sum(h[j] * h[j + 1] for j in range(len(h) - 1))
    return cfg["layers"] * per_layer


def storage_dtype(cfg):
    return F32 if cfg["dtype"] == "f32" else BF16


def tensor_specs(cfg, layer):
    """Recipe of one layer's parameters: name -> (shape, kind, stream id, mean, std, dtype).
    kind 'normal' draws mean + std * N(0,1); 'const' is the constant mean."""
    n, d, k, n_f, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_f"], cfg["n_l"]
    h = mlp_dims(cfg)
    wd = "f32" if cfg["dtype"] == "f32" else "bf16"
    specs = {
        "Y": ((n, k), "normal", layer_tid(layer, "Y"), 0.0, 1.0 / math.sqrt(n), wd),
        "W_L": ((n_l, n), "normal", layer_tid(layer, "W_L"), 0.0, 1.0 / math.sqrt(n), wd),
    }
    for j in range(len(h) - 1):
        specs["W%d" % j] = ((h[j + 1], h[j]), "normal", layer_tid(layer, "W", j), 0.0, 1.0 / math.sqrt(h[j]), wd)
        specs["b%d" % j] = ((h[j + 1],), "const", layer_tid(layer, "b", j), 0.0, 0.0, "f32")
    if cfg["ln_affine"] == "unit":
        specs["fmb_gamma"] = ((n * k,), "const", layer_tid(layer, "fmb_gamma"), 1.0, 0.0, "f32")
        specs["fmb_beta"] = ((n * k,), "const", layer_tid(layer, "fmb_beta"), 0.0, 0.0, "f32")
        specs["out_gamma"] = ((d,), "const", layer_tid(layer, "out_gamma"), 1.0, 0.0, "f32")
        specs["out_beta"] = ((d,), "const", layer_tid(layer, "out_beta"), 0.0, 0.0, "f32")
    else:  # 1 + N(0, 0.02^2) for every LayerNorm affine parameter
        for nm, size in (("fmb_gamma", n * k), ("fmb_beta", n * k), ("out_gamma", d), ("out_beta", d)):
            specs[nm] = ((size,), "normal", layer_tid(layer, nm), 1.0, 0.02, "f32")
    return specs


def make_layer_host(cfg, layer):
    """One layer's parameters as host numpy arrays (bf16 as uint16 bit patterns)."""
    out = {}
    for name, (shape, kind, tid, mean, std, dt) in tensor_specs(cfg, layer).items():
        if kind == "const":
            out[name] = np.full(shape, mean, dtype=np.float32) if dt == "f32" else None
            if out[name] is None:
                raise ValueError("bf16 constants are not used")
        else:
            arr = np.empty(shape, dtype=np.float32 if dt == "f32" else np.uint16)
            out[name] = fill_normal_host(arr, SEED, tid, mean, std)
    return out


def make_x_host(cfg, examples):
    """Rows X[b] for the listed example indices, as a host array [len(examples), n, d]
    (float32, or uint16 bf16 bits)."""
    n, d = cfg["n"], cfg["d"]
    per = n * d
    dt = np.float32 if cfg["dtype"] == "f32" else np.uint16
    out = np.empty((len(examples), n, d), dtype=dt)
    for r, b in enumerate(examples):
        row = out[r].reshape(-1)
        if cfg["x_dist"] == "logscaled":
            fill_x_logscaled_host(row, SEED, TID_X, TID_X_SCALE, n, d, offset=int(b) * per)
        else:
            fill_normal_host(row, SEED, TID_X, 0.0, 1.0, offset=int(b) * per)
    return out


def to_f64(arr):
    """Exact float64 view of a host tensor (float32 or bf16 bits)."""
    if arr.dtype == np.uint16:
        return bf16_bits_to_f64(arr).reshape(arr.shape)
    return arr.astype(np.float64)


def make_layer_dev(cfg, layer, device="cuda"):
    """One layer's parameters as device tensors, filled by the device generator
    (bit-identical to make_layer_host)."""
    import torch

    from . import fill_normal_dev
    out = {}
    for name, (shape, kind, tid, mean, std, dt) in tensor_specs(cfg, layer).items():
        tdt = torch.float32 if dt == "f32" else torch.bfloat16
        if kind == "const":
            out[name] = torch.full(shape, mean, dtype=tdt, device=device)
        else:
            t = torch.empty(shape, dtype=tdt, device=device)
            out[name] = fill_normal_dev(t, SEED, tid, mean, std)
    return out


def make_x_dev(cfg, batch, device="cuda", first_example=0):
    """X[first_example : first_example+batch] as a device tensor [batch, n, d]."""
    import torch

    from . import fill_normal_dev, fill_x_logscaled_dev
    n, d = cfg["n"], cfg["d"]
    tdt = torch.float32 if cfg["dtype"] == "f32" else torch.bfloat16
    t = torch.empty((batch, n, d), dtype=tdt, device=device)
    off = first_example * n * d
    if cfg["x_dist"] == "logscaled":
        fill_x_logscaled_dev(t, SEED, TID_X, TID_X_SCALE, n, d, offset=off)
    else:
        fill_normal_dev(t, SEED, TID_X, 0.0, 1.0, offset=off)
    return t


# ---------------------------------------------------------------- Wukong-MoE
#
# The Kunlun page (section 2.3, "Wukong Mixture of Experts") describes a global
# interaction module in which several Wukong modules run in parallel as the experts of
# one layer. Workloads of that form: each MoE layer holds E experts, each a Wukong layer
# of the shape below with its own weights, and a softmax gate over the experts computed
# from the flattened layer input. Gate weights W_g [E, n*d] ~ N(0, 1/(n*d)) and gate
# biases b_g [E] ~ N(0, 1) (non-zero so that the bias path is exercised); the experts'
# tensors follow the recipe of the plain workloads, each on its own streams.
MOE_CONFIGS = {
    "moe3_c2": dict(layers=2, experts=3, batch=2048, n=64, d=128, k=16, n_f=32, n_l=32, hidden=[1024],
                    dtype="bf16", ln_affine="1+N(0,0.02)", x_dist="normal",
                    about="2 MoE layers x 3 experts of the 2-layer bf16 shape, B=2048"),
    "moe4_c3": dict(layers=2, experts=4, batch=4096, n=256, d=160, k=32, n_f=128, n_l=128, hidden=[4096, 4096],
                    dtype="bf16", ln_affine="unit", x_dist="normal",
                    about="2 MoE layers x 4 experts of the 4-layer bf16 shape (n=256, d=160, k=32), B=4096"),
}


def expert_tid_offset(expert):
    """Stream-id offset of expert e's tensors (layer ids stay below 100 per layer)."""
    return 100 * (expert + 1)


def expert_specs(cfg, layer, expert):
    """Recipe of expert e of MoE layer `layer`: the plain layer recipe on shifted streams."""
    out = {}
    for name, (shape, kind, tid, mean, std, dt) in tensor_specs(cfg, layer).items():
        out[name] = (shape, kind, tid + expert_tid_offset(expert), mean, std, dt)
    return out


def gate_specs(cfg, layer):
    """Recipe of the gate of MoE layer `layer`: W_g [E, n*d], b_g [E] (fp32)."""
    E, nd = cfg["experts"], cfg["n"] * cfg["d"]
    wd = "f32" if cfg["dtype"] == "f32" else "bf16"
    base = 1000 * (layer + 1)
    return {"W_g": ((E, nd), "normal", base + 95, 0.0, 1.0 / math.sqrt(nd), wd),
            "b_g": ((E,), "normal", base + 96, 0.0, 1.0, "f32")}


def _host_from_specs(specs):
    out = {}
    for name, (shape, kind, tid, mean, std, dt) in specs.items():
        if kind == "const":
            if dt != "f32":
                raise ValueError("bf16 constants are not used")
            out[name] = np.full(shape, mean, dtype=np.float32)
        else:
            arr = np.empty(shape, dtype=np.float32 if dt == "f32" else np.uint16)
            out[name] = fill_normal_host(arr, SEED, tid, mean, std)
    return out


def _dev_from_specs(specs, device):
    import torch

    from . import fill_normal_dev
    out = {}
    for name, (shape, kind, tid, mean, std, dt) in specs.items():
        tdt = torch.float32 if dt == "f32" else torch.bfloat16
        if kind == "const":
            out[name] = torch.full(shape, mean, dtype=tdt, device=device)
        else:
            out[name] = fill_normal_dev(torch.empty(shape, dtype=tdt, device=device), SEED, tid, mean, std)
    return out


def make_expert_host(cfg, layer, expert):
    return _host_from_specs(expert_specs(cfg, layer, expert))


def make_expert_dev(cfg, layer, expert, device="cuda"):
    return _dev_from_specs(expert_specs(cfg, layer, expert), device)


def make_gate_host(cfg, layer):
    return _host_from_specs(gate_specs(cfg, layer))


def make_gate_dev(cfg, layer, device="cuda"):
    return _dev_from_specs(gate_specs(cfg, layer), device)


def moe_flops_per_example(cfg):
    """Matmul FLOPs of one example through the MoE stack: every expert's layer plus the
    gate's 2 * E * n * d per layer."""
    per_layer = flops_per_example(dict(cfg, layers=1))
    return cfg["layers"] * (cfg["experts"] * per_layer + 2 * cfg["experts"] * cfg["n"] * cfg["d"])


# ------------------------------------------------------------ prediction head
#
# The Wukong page (section 2.2) follows the stacked layers with an MLP that produces
# the prediction and gives it no sizes. The workloads' head: flatten (n*d) -> 1024 ->
# 256 -> 1 with ReLU between, T_j ~ N(0, 1/in_j), c_j ~ N(0, 0.1^2) (non-zero so the
# bias path is exercised), each tensor on its own stream.
HEAD_HIDDEN = [1024, 256]


def head_specs(cfg, hidden=None):
    hidden = HEAD_HIDDEN if hidden is None else list(hidden)
    dims = [cfg["n"] * cfg["d"]] + hidden + [1]
    wd = "f32" if cfg["dtype"] == "f32" else "bf16"
    specs = {}
    for j in range(len(dims) - 1):
        specs["T%d" % j] = ((dims[j + 1], dims[j]), "normal", 900000 + 10 * j, 0.0, 1.0 / math.sqrt(dims[j]), wd)
        specs["c%d" % j] = ((dims[j + 1],), "normal", 900000 + 10 * j + 1, 0.0, 0.1, "f32")
    return specs


def make_head_host(cfg, hidden=None):
    """[(T_j, c_j)] as host arrays (bf16 bits or float32)."""
    h = _host_from_specs(head_specs(cfg, hidden))
    return [(h["T%d" % j], h["c%d" % j]) for j in range(len(h) // 2)]


def make_head_dev(cfg, hidden=None, device="cuda"):
    h = _dev_from_specs(head_specs(cfg, hidden), device)
    return {"T": [h["T%d" % j] for j in range(len(h) // 2)], "c": [h["c%d" % j] for j in range(len(h) // 2)]}


def head_flops_per_example(cfg, hidden=None):
    hidden = HEAD_HIDDEN if hidden is None else list(hidden)
    dims = [cfg["n"] * cfg["d"]] + hidden + [1]
    return 2 * sum(dims[j] * dims[j + 1] for j in range(len(dims) - 1))


# ------------------------------------------------------- WHALE attention fusion
#
# WHALE pages (section 2.1 item 3, section 2.2): the Wukong representation H_w attends
# over the sequence representation H_s (K = V = H_s), the result is concatenated with
# H_w, projected by a fusion Linear and passed through a pre-norm shared-gate SwiGLU FFN.
# Workloads of that form: H_w stands for a Wukong stack's output (n x d per example, the
# shapes of the 2- and 8-layer workloads), H_s for an HSTU output of L positions (the
# pages scale L up to 15k); both synthetic N(0, 1). W_F [d, 2d], W_up [h, d], W_down [d, h]
# ~ N(0, 1/fan_in); b_F ~ N(0, 0.1^2); LayerNorm gamma = 1, beta = 0; h = 4d.
WHALE_CONFIGS = {
    "whale_c2": dict(batch=1024, n=64, d=128, L=2048, h=512, dtype="bf16",
                     about="n=64 queries of d=128 over L=2048, h=512, B=1024"),
    "whale_c4": dict(batch=256, n=512, d=160, L=4096, h=640, dtype="bf16",
                     about="n=512 queries of d=160 over L=4096, h=640, B=256"),
}

TID_WHALE_HW = 800001
TID_WHALE_HS = 800002


def whale_specs(cfg):
    d, h = cfg["d"], cfg["h"]
    return {"W_F": ((d, 2 * d), "normal", 800010, 0.0, 1.0 / math.sqrt(2 * d), "bf16"),
            "b_F": ((d,), "normal", 800011, 0.0, 0.1, "f32"),
            "ln_gamma": ((d,), "const", 800012, 1.0, 0.0, "f32"),
            "ln_beta": ((d,), "const", 800013, 0.0, 0.0, "f32"),
            "W_up": ((h, d), "normal", 800014, 0.0, 1.0 / math.sqrt(d), "bf16"),
            "W_down": ((d, h), "normal", 800015, 0.0, 1.0 / math.sqrt(h), "bf16")}


def make_whale_host(cfg):
    return _host_from_specs(whale_specs(cfg))


def make_whale_dev(cfg, device="cuda"):
    return _dev_from_specs(whale_specs(cfg), device)


def make_whale_inputs_host(cfg, examples):
    """(H_w [len, n, d], H_s [len, L, d]) as bf16 bit patterns for the listed examples."""
    n, L, d = cfg["n"], cfg["L"], cfg["d"]
    hw = np.empty((len(examples), n, d), dtype=np.uint16)
    hs = np.empty((len(examples), L, d), dtype=np.uint16)
    for r, b in enumerate(examples):
        fill_normal_host(hw[r].reshape(-1), SEED, TID_WHALE_HW, 0.0, 1.0, offset=int(b) * n * d)
        fill_normal_host(hs[r].reshape(-1), SEED, TID_WHALE_HS, 0.0, 1.0, offset=int(b) * L * d)
    return hw, hs


def make_whale_inputs_dev(cfg, batch, device="cuda", first_example=0):
    import torch

    from . import fill_normal_dev
    n, L, d = cfg["n"], cfg["L"], cfg["d"]
    hw = torch.empty((batch, n, d), dtype=torch.bfloat16, device=device)
    hs = torch.empty((batch, L, d), dtype=torch.bfloat16, device=device)
    fill_normal_dev(hw, SEED, TID_WHALE_HW, 0.0, 1.0, offset=first_example * n * d)
    fill_normal_dev(hs, SEED, TID_WHALE_HS, 0.0, 1.0, offset=first_example * L * d)
    return hw, hs


def whale_flops_per_example(cfg):
    """Matmul FLOPs of one example: 4 n L d (scores and weighted sum) + 2 n (2d) d (fusion)
    + 4 n d h (up and down)."""
    n, L, d, h = cfg["n"], cfg["L"], cfg["d"], cfg["h"]
    return 4 * n * L * d + 4 * n * d * d + 4 * n * d * h
