"""Times one step of the Wukong layer alone through its stand-alone C-ABI entry point.

    python microbench.py --kernel front|fm_ln|mlp_gemm|lcb|res_ln|moe_gate|moe_combine
        [--workload c4_bf16] [--batch B] [--iters K] [--dtype f16|bf16] [--layer-linear j] [--experts E]
    python microbench.py --kernel whale_attn|whale_ffn [--workload whale_c4] ...

Inputs are synthetic (the seeded generator), on the device, in the workload's
shapes. Prints one JSON line with the mean CUDA-event time per launch and the
algorithmic FLOPs / bytes of one launch. Small --iters values make it a convenient
target for a profiler capture of a single kernel.
"""
import argparse
import json
import os
import sys

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--kernel", required=True, choices=["front", "fm_ln", "mlp_gemm", "lcb", "res_ln", "moe_gate",
                                                           "moe_combine", "whale_attn", "whale_ffn"])
    ap.add_argument("--workload", default="c4_bf16")
    ap.add_argument("--batch", type=int, default=None)
    ap.add_argument("--iters", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--dtype", default="f16", choices=["f16", "bf16"])
    ap.add_argument("--layer-linear", type=int, default=0, help="which MLP Linear (mlp_gemm)")
    ap.add_argument("--no-affine", action="store_true", help="fm_ln without gamma/beta (as a stack runs it)")
    ap.add_argument("--experts", type=int, default=4, help="experts (moe_gate, moe_combine)")
    args = ap.parse_args()

    import torch

    import recsys_feature_interaction_b200 as wk
    from recsys_feature_interaction_b200 import build
    from synth import configs as C

    build.build()
    if args.kernel.startswith("whale"):
        run, flops, bytes_, B = _whale_case(args)
        return _time(args, run, flops, bytes_, B)
    if args.kernel == "front":
        return _front_case(args)
    cfg = C.MOE_CONFIGS[args.workload] if args.workload in C.MOE_CONFIGS else C.CONFIGS[args.workload]
    B = args.batch or cfg["batch"]
    n, d, k, n_f, n_l = cfg["n"], cfg["d"], cfg["k"], cfg["n_f"], cfg["n_l"]
    tdt = torch.float16 if args.dtype == "f16" else torch.bfloat16
    w = C.make_layer_dev(cfg, 0)
    dev = torch.device("cuda")
    X = C.make_x_dev(cfg, B).to(tdt)
    es = 2
    if args.kernel == "fm_ln":
        Y = w["Y"].to(tdt)
        A0 = torch.empty((B, n * k), dtype=tdt, device=dev)

        def run():
            wk.wk_fm_ln(X, Y, None if args.no_affine else w["fmb_gamma"], None if args.no_affine else w["fmb_beta"],
                        A0, B, n, d, k, args.dtype)
        flops = 4 * n * d * k * B
        bytes_ = (n * d + n * k) * es * B
    elif args.kernel == "mlp_gemm":
        dims = C.mlp_dims(cfg)
        j = args.layer_linear
        Kd, Nd = dims[j], dims[j + 1]
        A = torch.randn((B, Kd), device=dev).to(tdt)
        W = w["W%d" % j].to(tdt)
        Cm = torch.empty((B, Nd), dtype=tdt, device=dev)

        def run():
            wk.wk_mlp_linear(A, W, w["b%d" % j], Cm, B, Kd, Nd, Nd, j < len(dims) - 2, args.dtype)
        flops = 2 * B * Kd * Nd
        bytes_ = (B * Kd + Nd * Kd + B * Nd) * es
    elif args.kernel == "lcb":
        WL = w["W_L"].to(tdt)
        cat = torch.empty((B, n, d), dtype=tdt, device=dev)

        def run():
            wk.wk_lcb(WL, X, cat, B, n, d, n_f, n_l, args.dtype)
        flops = 2 * n_l * n * d * B
        bytes_ = (n * d + n_l * d) * es * B
    elif args.kernel == "moe_gate":
        E = args.experts
        Wg = (torch.randn((E, n * d), device=dev) / (n * d) ** 0.5).to(tdt)
        bg = torch.randn((E,), device=dev)
        g = torch.empty((B, E), device=dev)

        def run():
            wk.wk_moe_gate_softmax(X, Wg, bg, g, B, n * d, E, args.dtype)
        flops = 2 * E * n * d * B
        bytes_ = (n * d * es + E * 4) * B
    elif args.kernel == "moe_combine":
        E = args.experts
        cats = [torch.randn((B, n, d), device=dev).to(tdt) for _ in range(E)]
        g = torch.softmax(torch.randn((B, E), device=dev), dim=1)
        out = torch.empty_like(X)

        def run():
            wk.wk_moe_combine(cats, X, g, [w["out_gamma"]] * E, [w["out_beta"]] * E, out, B, n, d, args.dtype)
        flops = 0
        bytes_ = (E + 2) * n * d * es * B
    else:
        cat = torch.randn((B, n, d), device=dev).to(tdt)
        out = torch.empty_like(X)

        def run():
            wk.wk_res_ln(cat, X, w["out_gamma"], w["out_beta"], out, B * n, d, args.dtype)
        flops = 0
        bytes_ = 3 * n * d * es * B
    return _time(args, run, flops, bytes_, B)


def _front_case(args):
    """The one-kernel layer front (input LayerNorm, FM + LayerNorm, LCB, residual) of the
    workload's layer shape, inside a 2-layer stack whose FMB MLP is cut to one hidden width
    of 64 (the front does not depend on the MLP): layer 0's front converts the input, layer
    1's normalises the previous layer's output. Reports the mean of both layers' front
    launches from the stack's own per-kernel events; the workload's batch unless --batch."""
    import torch

    import recsys_feature_interaction_b200 as wk
    from synth import configs as C
    cfg = dict(C.CONFIGS[args.workload], layers=2, hidden=[64])
    B = args.batch or cfg["batch"]
    n, d, k = cfg["n"], cfg["d"], cfg["k"]
    layers = [C.make_layer_dev(cfg, l) for l in range(2)]
    h = wk.wk_stack_create(cfg, layers, max_batch=B)
    X = C.make_x_dev(cfg, B)
    out = torch.empty_like(X)
    for _ in range(args.warmup):
        wk.wk_stack_forward(h, X, out)
    torch.cuda.synchronize()
    wk.wk_stack_kernel_times(h)
    wk.wk_stack_set_profiling(h, True)
    for _ in range(args.iters):
        wk.wk_stack_forward(h, X, out)
    torch.cuda.synchronize()
    wk.wk_stack_set_profiling(h, False)
    t = wk.wk_stack_kernel_times(h)
    st = wk.wk_stack_sync_status(h)
    wk.wk_stack_destroy(h)
    ms_total, launches = t["front"]
    ms = ms_total / max(1, launches)
    flops = (4 * n * d * k + 2 * cfg["n_l"] * n * d) * B
    bytes_ = (2 * n * d + n * k) * 2 * B  # layer input in, layer output and A0 out (16-bit)
    print(json.dumps({"kernel": "front", "workload": args.workload, "batch": B, "dtype": "f16",
                      "ms_per_launch": ms, "launches": launches, "tflops": flops / (ms / 1e3) / 1e12,
                      "gbs": bytes_ / (ms / 1e3) / 1e9, "flops_per_launch": flops, "bytes_per_launch": bytes_,
                      "device_status": wk.wk_status_string(st)}))
    if st != wk.WK_OK:
        sys.exit(1)


def _whale_case(args):
    """The WHALE attention (A from H_w, H_s) or the fusion + FFN (H_f from H_w, A) alone."""
    import torch

    import recsys_feature_interaction_b200 as wk
    from synth import configs as C
    cfg = C.WHALE_CONFIGS[args.workload if args.workload in C.WHALE_CONFIGS else "whale_c4"]
    B = args.batch or cfg["batch"]
    n, L, d, h = cfg["n"], cfg["L"], cfg["d"], cfg["h"]
    tdt = torch.float16 if args.dtype == "f16" else torch.bfloat16
    Hw, Hs = C.make_whale_inputs_dev(cfg, B)
    Hw, Hs = Hw.to(tdt), Hs.to(tdt)
    A = torch.empty_like(Hw)
    es = 2
    if args.kernel == "whale_attn":
        def run():
            wk.wk_whale_attention(Hw, Hs, A, B, n, L, d, args.dtype)
        return run, 4 * n * L * d * B, (L * d + 2 * n * d) * es * B, B
    w = {k: (v.to(tdt) if v.dtype != torch.float32 else v) for k, v in C.make_whale_dev(cfg).items()}
    A.copy_(Hw * 0.5)
    Hf = torch.empty_like(Hw)
    rows = B * n

    def run():
        wk.wk_whale_fusion_ffn(Hw, A, w, Hf, rows, d, h, args.dtype)
    return run, rows * (4 * d * d + 4 * d * h), (3 * rows * d + 2 * d * d + 2 * d * h) * es, B


def _time(args, run, flops, bytes_, B):
    import torch

    import recsys_feature_interaction_b200 as wk
    for _ in range(args.warmup):
        run()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record()
    for _ in range(args.iters):
        run()
    e1.record()
    torch.cuda.synchronize()
    st = wk.wk_device_status()
    ms = e0.elapsed_time(e1) / max(1, args.iters)
    print(json.dumps({"kernel": args.kernel, "workload": args.workload, "batch": B, "dtype": args.dtype,
                      "ms_per_launch": ms, "tflops": flops / (ms / 1e3) / 1e12 if flops else None,
                      "gbs": bytes_ / (ms / 1e3) / 1e9, "flops_per_launch": flops, "bytes_per_launch": bytes_,
                      "device_status": wk.wk_status_string(st)}))
    if st != wk.WK_OK:
        sys.exit(1)


if __name__ == "__main__":
    main()
