"""Throughput of the Wukong interaction-stack forward on B200s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--workload NAME]
    (N > 1: python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N ...)

One step is one forward of the whole stack (every layer: FM + LayerNorm, the FMB
MLP, the LCB, residual + LayerNorm) over one batch of synthetic examples. The
workload is the 8-layer bf16 stack (n=512 embeddings, d=160, k=64, n_F=n_L=256,
FMB MLP 32768->16384->16384->40960, ~24.1 GFLOP/example) at batch 4096 per GPU;
--workload names one of the other synthetic workloads (synth/configs.py) instead.
Several GPUs run independent replicas on disjoint batches (the examples are
independent, so there is no collective in the forward): weak scaling.

Rank 0 prints one JSON line. `value` is examples/s of the whole job with the
inputs resident in HBM (CUDA events on the launch stream, max over ranks);
`e2e` is the same metric through the public forward with pinned host buffers
(every step's host-to-device copy of X and device-to-host copy of the output inside
the timed region): for a stack, the streamed host forward
(wk_stack_forward_host_async, a serving loop that waits for step i-1's result after
issuing step i), with the synchronous wk_stack_forward_host beside it in
`e2e.synchronous_call`; `roofline` reports the MLP GEMM kernel (the dominant one)
against the measured bf16 peak; `cpu_baseline` times the fp64 oracle on a bounded
sample.
"""
import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

WORKLOAD = "c4_bf16"
METRIC = "examples/sec and achieved TFLOP/s (% of bf16 peak), Wukong stack fwd, 1 B200"
# examples per oracle sample (one layer), sized for a few seconds of host work each
ORACLE_SAMPLE = {"c1_fp32": 64, "c2_bf16": 4096, "c3_bf16": 128, "c4_bf16": 16, "c5_bf16": 512, "moe3_c2": 1024,
                 "moe4_c3": 32, "whale_c2": 512, "whale_c4": 32}
WHALE_METRIC = "examples/sec and achieved TFLOP/s (% of bf16 peak), WHALE attention fusion fwd, 1 B200"
BACKWARD_METRIC = ("examples/sec and achieved TFLOP/s (% of bf16 peak), Wukong stack training step "
                   "(forward + backward: gradients of the input and of every parameter), 1 B200")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


# DRAM traffic of the CTA-pair MLP GEMM per launch, from one ncu capture of the three Linears
# of the first layer inside the bench's own step (dram__bytes_read.sum + dram__bytes_write.sum,
# averaged over the three launches; the last Linear reduce-adds into the layer output, so its
# output is read as well as written). It describes the kernel sources it was taken on: when
# their hash differs, the bench reports null.
GEMM_TRAFFIC = {
    "sources": ["recsys_feature_interaction_b200/csrc/gemm_tc2.cuh", "recsys_feature_interaction_b200/csrc/common.cuh"],
    "sha256": "c5d76cd63c37947785bb77b92b43359c5a3e9b9f076ba31087abab135dce9d9b",
    "bytes_per_launch": 3338665301,
}


def sources_sha256(paths):
    import hashlib
    h = hashlib.sha256()
    for rel in paths:
        with open(os.path.join(ROOT, rel), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def gemm_traffic():
    """DRAM bytes per MLP GEMM launch from the committed capture, or None when the
    kernel sources have changed since."""
    if GEMM_TRAFFIC["bytes_per_launch"] is None or GEMM_TRAFFIC["sha256"] != sources_sha256(GEMM_TRAFFIC["sources"]):
        return None
    return GEMM_TRAFFIC["bytes_per_launch"]


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def workload_desc(cfg):
    if "L" in cfg:
        return ("WHALE attention fusion fwd, %s: n=%d queries of d=%d over L=%d shared keys/values, fusion "
                "Linear %d->%d, pre-norm shared-gate SwiGLU %d->%d->%d" %
                (cfg["dtype"], cfg["n"], cfg["d"], cfg["L"], 2 * cfg["d"], cfg["d"], cfg["d"], cfg["h"], cfg["d"]))
    dims = [cfg["n"] * cfg["k"]] + list(cfg["hidden"]) + [cfg["n_f"] * cfg["d"]]
    kind = ("Wukong-MoE stack fwd (%d experts per layer, softmax gate)" % cfg["experts"] if "experts" in cfg
            else "Wukong stack fwd")
    return ("%d-layer %s %s: n=%d, d=%d, k=%d, n_F=n_L=%d, FMB MLP %s" %
            (cfg["layers"], cfg["dtype"], kind, cfg["n"], cfg["d"], cfg["k"], cfg["n_f"],
             "->".join(str(v) for v in dims)))


def fp32_alu_peak(peaks):
    """fp32 CUDA-core peak of the GPU (TFLOP/s): 148 SMs x 128 FMA lanes x 2 FLOP x the
    SM clock (the measured max clock from the peaks file, else 1965 MHz)."""
    mhz = peaks.get("sm_max_mhz") or 1965.0
    return 148 * 128 * 2 * mhz * 1e6 / 1e12


def gemm_flops_per_example(cfg):
    dims = [cfg["n"] * cfg["k"]] + list(cfg["hidden"]) + [cfg["n_f"] * cfg["d"]]
    return cfg["layers"] * 2 * sum(dims[j] * dims[j + 1] for j in range(len(dims) - 1))


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms while running."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index):
        self.gpu = gpu_index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.QUERY,
                                          "--format=csv,noheader,nounits", "-lms", "200"],
                                         stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.lines = []
        if self.proc is not None:
            time.sleep(0.25)
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, pw, mx, reasons = [], [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            try:
                pw.append(float(f[3]))
            except ValueError:
                pass
            for nm, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(nm)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": mx, "reasons": [], "samples": 0}
        loaded = [v for v in sm if mx is None or v > 0.3 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": sorted(reasons),
                "samples": len(sm), "power_w": statistics.median(pw) if pw else None}


def oracle_sample(cfg, n_examples, threads=None):
    """Times the fp64 oracle on n_examples examples through ONE layer (the layer's
    weights are generated before the clock starts) and returns (examples/s of the
    whole stack, seconds, threads)."""
    import oracle
    from synth import configs as C
    if "L" in cfg:  # WHALE fusion: numpy fp64 per example (BLAS threads)
        from threadpoolctl import threadpool_info
        hw, hs = C.make_whale_inputs_host(cfg, list(range(n_examples)))
        hw, hs = C.to_f64(hw), C.to_f64(hs)
        w = C.make_whale_host(cfg)
        t0 = time.perf_counter()
        for b in range(n_examples):
            oracle.whale_fusion(hw[b], hs[b], w)
        dt = time.perf_counter() - t0
        thr = max([p.get("num_threads", 1) for p in threadpool_info()] or [1])
        return n_examples / dt, dt, thr
    X = C.to_f64(C.make_x_host(cfg, list(range(n_examples))))
    thr = threads or oracle.default_threads()
    if "experts" in cfg:
        experts = [C.make_expert_host(cfg, 0, e) for e in range(cfg["experts"])]
        gate = C.make_gate_host(cfg, 0)
        t0 = time.perf_counter()
        oracle.moe_layer_forward(cfg, experts, gate, X, threads=thr)
    else:
        w = C.make_layer_host(cfg, 0)
        t0 = time.perf_counter()
        oracle.layer_forward(cfg, w, X, threads=thr)
    dt = time.perf_counter() - t0
    return n_examples / (dt * cfg["layers"]), dt, thr


def backward_oracle_sample(cfg, n_examples, dO=None):
    """Times the fp64 oracle's forward and backward of ONE layer on n_examples examples
    (weights, inputs and the upstream gradient made before the clock starts) and returns
    (examples/s of the whole stack's training step, seconds, threads)."""
    import numpy as np
    from threadpoolctl import threadpool_info

    import oracle
    from synth import configs as C
    Xh = C.to_f64(C.make_x_host(cfg, list(range(n_examples))))
    w = C.make_layer_host(cfg, 0)
    if dO is None:
        dO = np.random.RandomState(1234).standard_normal(Xh.shape)
    t0 = time.perf_counter()
    oracle.layer_backward(cfg, w, Xh, dO)
    dt = time.perf_counter() - t0
    thr = max([pp.get("num_threads", 1) for pp in threadpool_info()] or [1])
    return n_examples / (dt * cfg["layers"]), dt, thr


def backward_sample_size(workload):
    return max(1, min(16, ORACLE_SAMPLE.get(workload, 16) // 8))


def workload_cfg(name):
    from synth import configs as C
    if name in C.WHALE_CONFIGS:
        return C.WHALE_CONFIGS[name]
    return C.MOE_CONFIGS[name] if name in C.MOE_CONFIGS else C.CONFIGS[name]


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on the host cores."""
    if rank != 0:
        return
    cfg = workload_cfg(args.workload)
    whale = "L" in cfg
    backward = args.backward and not whale and "experts" not in cfg
    vals = []
    ns = backward_sample_size(args.workload) if backward else ORACLE_SAMPLE[args.workload]
    sample_fn = backward_oracle_sample if backward else oracle_sample
    for _ in range(args.warmup):
        sample_fn(cfg, ns)
    thr = None
    for _ in range(args.steps):
        v, dt, thr = sample_fn(cfg, ns)
        vals.append(v)
    value = statistics.median(vals)
    if whale:
        sample = "%d examples of the fusion per step" % ns
    elif backward:
        sample = ("%d examples through the forward and backward of 1 of the %d layers per step (numpy "
                  "float64), scaled to the whole stack" % (ns, cfg["layers"]))
    else:
        sample = "%d examples through 1 of the %d layers per step, scaled to the whole stack" % (ns, cfg["layers"])
    metric = WHALE_METRIC if whale else (BACKWARD_METRIC if backward else METRIC)
    line = {"impl": "reference", "metric": metric, "value": value, "unit": "examples/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload + ": " + workload_desc(cfg) + (", training step" if backward else ""),
                       "global_batch": cfg["batch"],
                       "oracle": ("numpy fp64 (BLAS threads)" if whale or backward else
                                  "plain C fp64, threads over examples / output rows")},
            "cpu_baseline": {"value": value, "unit": "examples/s", "cores": thr, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "examples/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def run_whale(args, cfg, rank, world, local, dev):
    """One step = one WHALE fusion forward (attention with shared K = V, fusion Linear,
    pre-norm shared-gate SwiGLU FFN) over the per-GPU batch; roofline on the attention
    kernel (tensor-bound when 2 * L * d * n / (L * d * 2) = 2n FLOP per H_s byte is above
    the ridge, else HBM-bound)."""
    import torch

    import recsys_feature_interaction_b200 as wk
    from recsys_feature_interaction_b200 import replicas
    from synth import configs as C

    B, n, L, d = cfg["batch"], cfg["n"], cfg["L"], cfg["d"]
    first, _ = replicas.example_range(rank, world, B)
    Hw, Hs = C.make_whale_inputs_dev(cfg, B, device=dev, first_example=first)
    Hf = torch.empty_like(Hw)
    w = C.make_whale_dev(cfg, device=dev)
    h = wk.wk_whale_create(cfg, w, max_batch=B)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        wk.wk_whale_forward(h, Hw, Hs, Hf, stream=stream)
    torch.cuda.synchronize(dev)
    if wk.wk_whale_sync_status(h) != wk.WK_OK:
        raise RuntimeError("device status after warm-up")
    wk.wk_whale_kernel_times(h)  # clear
    in_bytes = (Hw.numel() + Hs.numel()) * Hw.element_size()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < (252 << 20) else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps if flush is not None else 1)]
    replicas.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        if flush is None:
            evs[0][0].record(stream)
            for _ in range(args.steps):
                wk.wk_whale_forward(h, Hw, Hs, Hf, stream=stream)
            evs[0][1].record(stream)
        else:
            for a, b in evs:
                flush.fill_(1)
                a.record(stream)
                wk.wk_whale_forward(h, Hw, Hs, Hf, stream=stream)
                b.record(stream)
        torch.cuda.synchronize(dev)
    replicas.barrier()
    ms = sum(a.elapsed_time(b) for a, b in evs)
    if wk.wk_whale_sync_status(h) != wk.WK_OK:
        raise RuntimeError("device status after the timed region")
    # per-kernel times from a second, profiled pass of the same steps
    wk.wk_whale_set_profiling(h, True)
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        wk.wk_whale_forward(h, Hw, Hs, Hf, stream=stream)
    torch.cuda.synchronize(dev)
    wk.wk_whale_set_profiling(h, False)
    ktimes = wk.wk_whale_kernel_times(h)
    ms_max = replicas.max_over_ranks(ms, device=dev)
    value = world * B * args.steps / (ms_max / 1e3)

    # end to end: H_w and H_s copied in from pinned host memory, H_f copied out, every step
    hwh, hsh = Hw.cpu().pin_memory(), Hs.cpu().pin_memory()
    hfh = torch.empty_like(Hf, device="cpu").pin_memory()

    def fwd_host():
        Hw.copy_(hwh, non_blocking=True)
        Hs.copy_(hsh, non_blocking=True)
        wk.wk_whale_forward(h, Hw, Hs, Hf, stream=stream)
        hfh.copy_(Hf, non_blocking=True)
        stream.synchronize()
    fwd_host()
    replicas.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fwd_host()
    e2e_s = replicas.max_over_ranks(time.perf_counter() - t0, device=dev)
    e2e_value = world * B * args.steps / e2e_s

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops_ex = C.whale_flops_per_example(cfg)
        tflops = value * flops_ex / 1e12 / world
        a_ms, a_n = ktimes["whale_attn"]
        a_s = (a_ms / a_n) / 1e3 if a_n else None
        attn_flops = 4.0 * n * L * d * B                           # per launch: S = Q K^T and P V
        attn_bytes = float(B) * (L * d + 2 * n * d) * 2            # H_s once, H_w in, A out
        ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
        if attn_flops / attn_bytes >= ridge:
            ach = attn_flops / a_s / 1e12 if a_s else None
            roof = {"kernel": "whale_attn_kernel (tcgen05)", "bound": "tensor", "achieved": ach,
                    "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                    "peak_note": "%s burst cuBLAS bf16 (a kernel of well under a second)" % peak_src}
        else:
            ach = attn_bytes / a_s / 1e9 if a_s else None
            roof = {"kernel": "whale_attn_kernel (tcgen05)", "bound": "hbm", "achieved": ach,
                    "peak": peaks["hbm_gbs"], "unit": "GB/s", "peak_note": "%s copy bandwidth" % peak_src}
        roof["frac"] = (ach / roof["peak"]) if ach else None
        roof["traffic"] = None
        roof["algorithmic_per_launch"] = {"flops": attn_flops, "bytes": attn_bytes}
        l2 = ("L2 flushed (256 MB write) before every step, outside the timed events" if flush is not None else
              "inputs larger than L2 (H_w + H_s %.0f MB per GPU)" % (in_bytes / 1e6))
        line = {
            "metric": WHALE_METRIC, "value": value, "unit": "examples/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": cfg["dtype"], "data": "synthetic",
            "config": {"workload": args.workload + ": " + workload_desc(cfg), "per_gpu_batch": B,
                       "precision": "16-bit inputs, weights, softmax weights and gated activations; fp32 "
                                    "accumulation, softmax and LayerNorm statistics",
                       "global_batch": B * world, "seq_len": L, "parallelism": "replicas (batch shards)",
                       "l2": l2, "launch": "eager, one C-ABI call per step"},
            "tflops_per_gpu": tflops,
            "pct_of_bf16_peak": 100.0 * tflops / peaks["bf16_tflops"],
            "peak_source": "%s bf16_tflops (burst)" % peak_src,
            "roofline": roof,
            "kernel_ms_per_step": {k: v[0] / args.steps for k, v in ktimes.items() if v[1]},
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": "examples/s",
                    "h2d_bytes_per_step": in_bytes, "d2h_bytes_per_step": Hf.numel() * Hf.element_size(),
                    "api": "wk_whale_forward with pinned host-to-device copies of H_w and H_s before and a "
                           "device-to-host copy of H_f after"},
            "gpu_launches": sum(v[1] for v in ktimes.values()),
        }
        if world == 1 and not args.no_cpu_baseline:
            ns = ORACLE_SAMPLE[args.workload]
            v, dt, thr = oracle_sample(cfg, ns)
            line["cpu_baseline"] = {"value": v, "unit": "examples/s", "cores": thr, "kind": "oracle",
                                    "sample": "%d examples of the fusion (%.1f s)" % (ns, dt)}
        print(json.dumps(line), flush=True)
    wk.wk_whale_destroy(h)


def run_backward(args, cfg, rank, world, local, dev):
    """One step = wk_stack_backward over the per-GPU batch: the forward with every layer's
    input and activations saved, then each layer differentiated (dX and all parameter
    gradients). Algorithmic work: 3x the forward's matmul FLOPs. Roofline: the FMB MLP GEMM
    (forward, input and weight gradients), tensor-bound."""
    import torch

    import recsys_feature_interaction_b200 as wk
    from recsys_feature_interaction_b200 import replicas
    from synth import configs as C

    B, L, n, d, k = cfg["batch"], cfg["layers"], cfg["n"], cfg["d"], cfg["k"]
    dims = C.mlp_dims(cfg)
    first, _ = replicas.example_range(rank, world, B)
    X = C.make_x_dev(cfg, B, device=dev, first_example=first)
    layers = [C.make_layer_dev(cfg, l, device=dev) for l in range(L)]
    h = wk.wk_stack_create(cfg, layers, max_batch=B)
    gen = torch.Generator(device=dev)
    gen.manual_seed(1234 + rank)
    dOut = torch.randn((B, n, d), generator=gen, device=dev, dtype=torch.float32)
    dX = torch.empty_like(dOut)
    # the gradients in one flat buffer per layer; with several ranks every step ends with
    # their average over the ranks (NCCL), layer l's all-reduce on a side stream as soon as
    # the backward has recorded layer l's event
    buckets = replicas.GradBuckets(n, d, k, cfg["n_l"], dims, L, device=dev)
    grads = buckets.grads
    stream = torch.cuda.current_stream(dev)
    comm = torch.cuda.Stream(dev) if world > 1 else None
    layer_ev = [torch.cuda.Event() for _ in range(L)] if world > 1 else None

    def train_step():
        wk.wk_stack_backward(h, X, dOut, dX, grads, stream=stream, layer_events=layer_ev)
        if world > 1:
            replicas.average_gradients(buckets.flats, layer_ev, comm)

    for _ in range(args.warmup):
        train_step()
    torch.cuda.synchronize(dev)
    if wk.wk_stack_sync_status(h) != wk.WK_OK:
        raise RuntimeError("device status after warm-up")
    wk.wk_stack_kernel_times(h)  # clear
    in_bytes = X.numel() * X.element_size() + dOut.numel() * 4
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if in_bytes < (252 << 20) else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps if flush is not None else 1)]
    replicas.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        if flush is None:
            evs[0][0].record(stream)
            for _ in range(args.steps):
                train_step()
            evs[0][1].record(stream)
        else:
            for a, b in evs:
                flush.fill_(1)
                a.record(stream)
                train_step()
                b.record(stream)
        torch.cuda.synchronize(dev)
    replicas.barrier()
    ms = sum(a.elapsed_time(b) for a, b in evs)
    if wk.wk_stack_sync_status(h) != wk.WK_OK:
        raise RuntimeError("device status after the timed region")
    # per-kernel times from a second, profiled pass of the same steps
    wk.wk_stack_set_profiling(h, True)
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        train_step()
    torch.cuda.synchronize(dev)
    wk.wk_stack_set_profiling(h, False)
    ktimes = wk.wk_stack_kernel_times(h)
    ms_max = replicas.max_over_ranks(ms, device=dev)
    value = world * B * args.steps / (ms_max / 1e3)

    # end to end: X and dOut copied in from pinned host memory, dX copied out, every step
    xh, dh = X.cpu().pin_memory(), dOut.cpu().pin_memory()
    dxh = torch.empty_like(dX, device="cpu").pin_memory()

    def step_host():
        X.copy_(xh, non_blocking=True)
        dOut.copy_(dh, non_blocking=True)
        train_step()
        dxh.copy_(dX, non_blocking=True)
        stream.synchronize()
    step_host()
    replicas.barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step_host()
    e2e_value = world * B * args.steps / replicas.max_over_ranks(time.perf_counter() - t0, device=dev)

    if rank == 0:
        peaks, peak_src = load_peaks()
        fwd = C.flops_per_example(cfg)
        flops_ex = 3 * fwd
        tflops = value * flops_ex / 1e12 / world
        # executed MLP GEMM work per step: the forward (L layers, activations saved, none
        # recomputed) and the input and weight gradients (2 L), each the forward's per-layer
        # MLP FLOPs
        mlp_layer = gemm_flops_per_example(cfg) / L * B
        gemm_flops_step = 3 * L * mlp_layer
        g_ms, g_n = ktimes["mlp_gemm"]
        ach = gemm_flops_step * args.steps / (g_ms / 1e3) / 1e12 if g_ms else None
        peak = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
        roof = {"kernel": "mlp_gemm (tcgen05 pair GEMM: forward, input and weight gradients, the gradients reading MN-major operands)", "bound": "tensor",
                "achieved": ach, "peak": peak, "unit": "TFLOP/s", "frac": (ach / peak) if ach else None,
                "traffic": None, "peak_note": "%s sustained cuBLAS bf16" % peak_src,
                "algorithmic_per_step": {"flops": gemm_flops_step, "launches": g_n / max(1, args.steps)}}
        l2 = ("L2 flushed (256 MB write) before every step, outside the timed events" if flush is not None else
              "inputs larger than L2 (X and dOut %.0f MB per GPU)" % (in_bytes / 1e6))
        line = {
            "metric": BACKWARD_METRIC, "value": value, "unit": "examples/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "config": {"workload": args.workload + ": " + workload_desc(cfg) + ", training step", "per_gpu_batch": B,
                       "precision": "bf16 inputs and weights; fp16 tensor-core operands, activations and MLP "
                                    "gradients; fp32 accumulation, LayerNorm statistics, layer-stream and "
                                    "parameter gradients",
                       "global_batch": B * world, "seq_len": None,
                       "parallelism": ("dp%d: batch shards, parameter gradients averaged over the ranks (NCCL "
                                       "all-reduce per layer, overlapped with the backward of the layers below)"
                                       % world) if world > 1 else "one GPU",
                       "l2": l2, "launch": "eager, one C-ABI call per step",
                       "flops_per_example": "3 x forward matmul FLOPs = %.4g" % flops_ex},
            "tflops_per_gpu": tflops,
            "pct_of_bf16_peak": 100.0 * tflops / peak,
            "peak_source": "%s bf16_tflops_sustained" % peak_src,
            "roofline": roof,
            "kernel_ms_per_step": {kk: v[0] / args.steps for kk, v in ktimes.items() if v[1]},
            "clocks": clk.summary(),
            "e2e": {"value": e2e_value, "unit": "examples/s", "h2d_bytes_per_step": in_bytes,
                    "d2h_bytes_per_step": dX.numel() * 4,
                    "api": "wk_stack_backward with pinned host-to-device copies of X and dOut before and a "
                           "device-to-host copy of dX after (parameter gradients stay on the device)"},
            "gpu_launches": sum(v[1] for v in ktimes.values()),
        }
        if world == 1 and not args.no_cpu_baseline:
            ns = backward_sample_size(args.workload)
            v, dt, thr = backward_oracle_sample(cfg, ns, dOut[:ns].double().cpu().numpy())
            line["cpu_baseline"] = {"value": v, "unit": "examples/s", "cores": thr, "kind": "oracle",
                                    "sample": "%d examples through the forward and backward of 1 of the %d layers "
                                              "(%.1f s, numpy float64), scaled to the stack" % (ns, L, dt)}
        print(json.dumps(line), flush=True)
    wk.wk_stack_destroy(h)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--graph", action="store_true",
                    help="replay each step from a CUDA graph of one forward (wk_*_graph_create); the "
                         "per-kernel times then come from an eager profiled pass after the timed region")
    ap.add_argument("--head", action="store_true",
                    help="each step also runs the prediction head (wk_stack_predict: logits and probabilities)")
    ap.add_argument("--backward", action="store_true",
                    help="each step is a training step: wk_stack_backward (forward with saved layer inputs, "
                         "then the gradients of the input and of every parameter)")
    ap.add_argument("--workload", default=WORKLOAD,
                    choices=["c1_fp32", "c2_bf16", "c3_bf16", "c4_bf16", "c5_bf16", "moe3_c2", "moe4_c3",
                             "whale_c2", "whale_c4"])
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)

    from recsys_feature_interaction_b200 import replicas

    rank, world, local = replicas.rank_info()

    if args.impl == "reference":
        run_reference(args, rank, world)
        return

    import torch

    import recsys_feature_interaction_b200 as wk
    from recsys_feature_interaction_b200 import build as wk_build
    from synth import configs as C

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    replicas.init("nccl", device=dev)
    wk_build.build()

    cfg = workload_cfg(args.workload)
    if "L" in cfg:
        run_whale(args, cfg, rank, world, local, dev)
        replicas.finish()
        return
    if args.backward:
        run_backward(args, cfg, rank, world, local, dev)
        replicas.finish()
        return
    moe = "experts" in cfg
    host_stream = None
    B = cfg["batch"]
    # rank r works on examples [r*B, (r+1)*B) of the synthetic stream (no collective on the data path)
    first, _ = replicas.example_range(rank, world, B)
    X = C.make_x_dev(cfg, B, device=dev, first_example=first)
    out = torch.empty_like(X)
    stream = torch.cuda.current_stream(dev)
    if moe:
        params = [[C.make_expert_dev(cfg, l, e, device=dev) for e in range(cfg["experts"])]
                  for l in range(cfg["layers"])]
        gates = [C.make_gate_dev(cfg, l, device=dev) for l in range(cfg["layers"])]
        h = wk.wk_moe_create(cfg, params, gates, max_batch=B)
        api = dict(fwd=lambda x, o: wk.wk_moe_forward(h, x, o, stream=stream),
                   status=lambda: wk.wk_moe_sync_status(h), prof=lambda on: wk.wk_moe_set_profiling(h, on),
                   times=lambda: wk.wk_moe_kernel_times(h), destroy=lambda: wk.wk_moe_destroy(h))
        w_tensors = [t for lay in params for ex in lay for t in ex.values()] + \
                    [t for g in gates for t in g.values()]
        flops_ex = C.moe_flops_per_example(cfg)

        def fwd_host(xh, oh):  # the public forward with the step's input and result on the host
            X.copy_(xh, non_blocking=True)
            api["fwd"](X, out)
            oh.copy_(out, non_blocking=True)
            stream.synchronize()
        e2e_api = "wk_moe_forward with a pinned host-to-device copy before and device-to-host copy after"
    elif args.head:
        layers = [C.make_layer_dev(cfg, l, device=dev) for l in range(cfg["layers"])]
        h = wk.wk_stack_create(cfg, layers, max_batch=B)
        head = C.make_head_dev(cfg, device=dev)
        wk.wk_stack_set_head(h, head)
        logit = torch.empty((B,), device=dev)
        prob = torch.empty((B,), device=dev)
        api = dict(fwd=lambda x, o: wk.wk_stack_predict(h, x, logit, prob, stream=stream),
                   status=lambda: wk.wk_stack_sync_status(h), prof=lambda on: wk.wk_stack_set_profiling(h, on),
                   times=lambda: wk.wk_stack_kernel_times(h), destroy=lambda: wk.wk_stack_destroy(h))
        w_tensors = [t for lw in layers for t in lw.values()] + list(head["T"]) + list(head["c"])
        flops_ex = C.flops_per_example(cfg) + C.head_flops_per_example(cfg)
        out = prob

        def fwd_host(xh, oh):  # input copied in, the probabilities copied out
            X.copy_(xh, non_blocking=True)
            api["fwd"](X, None)
            oh.copy_(prob, non_blocking=True)
            stream.synchronize()
        e2e_api = "wk_stack_predict with a pinned host-to-device copy of X and a device-to-host copy of prob"
    else:
        layers = [C.make_layer_dev(cfg, l, device=dev) for l in range(cfg["layers"])]
        h = wk.wk_stack_create(cfg, layers, max_batch=B)
        api = dict(fwd=lambda x, o: wk.wk_stack_forward(h, x, o, stream=stream),
                   status=lambda: wk.wk_stack_sync_status(h), prof=lambda on: wk.wk_stack_set_profiling(h, on),
                   times=lambda: wk.wk_stack_kernel_times(h), destroy=lambda: wk.wk_stack_destroy(h))
        w_tensors = [t for lw in layers for t in lw.values()]
        flops_ex = C.flops_per_example(cfg)

        def fwd_host(xh, oh):
            wk.wk_stack_forward_host(h, xh, oh)
        e2e_api = "wk_stack_forward_host (chunked copies overlapped with compute)"

        def host_stream(xhs, ohs, steps):
            # a serving loop: step i's input copy, forward and output copy are enqueued,
            # then step i-1's result is waited for on the host
            prev = None
            for i in range(steps):
                t = wk.wk_stack_forward_host_async(h, xhs[i % 2], ohs[i % 2])
                if prev is not None:
                    wk.wk_stack_host_wait(h, prev)
                prev = t
            wk.wk_stack_host_wait(h)
        stream_api = ("wk_stack_forward_host_async + wk_stack_host_wait, a serving loop over two pairs of "
                      "page-locked host buffers: step i+1's input copy and step i-1's output copy run while "
                      "step i's forward computes, the whole batch per forward")

    barrier = replicas.barrier

    def max_over_ranks(v):
        return replicas.max_over_ranks(v, device=dev)

    for _ in range(args.warmup):
        api["fwd"](X, out)
    torch.cuda.synchronize(dev)
    if api["status"]() != wk.WK_OK:
        raise RuntimeError("device status after warm-up")
    api["times"]()  # clear

    # ---- device-resident timing. A workload whose input is smaller than twice the
    # L2 (126 MB) gets an L2 flush (a 256 MB write) before every step, outside the
    # per-step event pairs; larger inputs stream through L2 by themselves.
    x_bytes = X.numel() * X.element_size()
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev) if x_bytes < (252 << 20) else None
    graph = None
    step = api["fwd"]
    if args.graph:
        if args.head:
            raise SystemExit("--graph captures wk_stack_forward / wk_moe_forward, not the head")
        graph = (wk.wk_moe_graph_create if moe else wk.wk_stack_graph_create)(h, X, out)
        wk.wk_graph_launch(graph, stream)  # warm the graph

        def step(x, o):
            wk.wk_graph_launch(graph, stream)
    # the timed steps run with the library's per-kernel events off; the per-kernel split
    # (and the roofline's kernel time) comes from a second, profiled pass of the same steps
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps if flush is not None else 1)]
    barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(local) as clk:
        if flush is None:
            evs[0][0].record(stream)
            for _ in range(args.steps):
                step(X, out)
            evs[0][1].record(stream)
        else:
            for a, b in evs:
                flush.fill_(1)
                a.record(stream)
                step(X, out)
                b.record(stream)
        torch.cuda.synchronize(dev)
    barrier()
    ms = sum(a.elapsed_time(b) for a, b in evs)
    status = api["status"]()
    if status != wk.WK_OK:
        raise RuntimeError("device status: " + wk.wk_status_string(status))
    # per-kernel times: an eager profiled pass of the same steps (the library records a CUDA
    # event pair around every launch on the launch stream)
    api["prof"](True)
    for _ in range(args.steps):
        if flush is not None:
            flush.fill_(1)
        api["fwd"](X, out)
    torch.cuda.synchronize(dev)
    api["prof"](False)
    if graph is not None:
        wk.wk_graph_destroy(graph)
    ktimes = api["times"]()
    ms_max = max_over_ranks(ms)
    value = world * B * args.steps / (ms_max / 1e3)

    # ---- end to end with host buffers
    xh = X.cpu().pin_memory()
    oh = torch.empty_like(out, device="cpu").pin_memory()
    fwd_host(xh, oh)  # warm the staging buffers
    barrier()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        fwd_host(xh, oh)
    e2e_s = max_over_ranks(time.perf_counter() - t0)
    e2e_value = world * B * args.steps / e2e_s
    e2e_sync = None
    if host_stream is not None:
        # the next batch of this rank's examples as the second host input
        x2 = C.make_x_dev(cfg, B, device=dev, first_example=first + world * B)
        xhs = [xh, x2.cpu().pin_memory()]
        del x2
        ohs = [oh, torch.empty_like(oh).pin_memory()]
        host_stream(xhs, ohs, 2)  # warm the slots
        barrier()
        t0 = time.perf_counter()
        host_stream(xhs, ohs, args.steps)
        s_s = max_over_ranks(time.perf_counter() - t0)
        e2e_sync = {"value": e2e_value, "api": e2e_api}
        e2e_value, e2e_api = world * B * args.steps / s_s, stream_api
    step_bytes = B * cfg["n"] * cfg["d"] * X.element_size()
    out_bytes = oh.numel() * oh.element_size()

    if rank == 0:
        peaks, peak_src = load_peaks()
        tflops = value * flops_ex / 1e12 / world
        g_ms, g_n = ktimes["mlp_gemm"]
        gemm_flops_launch = gemm_flops_per_example(cfg) * B / (cfg["layers"] * (len(cfg["hidden"]) + 1))
        achieved = gemm_flops_launch / ((g_ms / g_n) / 1e3) / 1e12 if g_n else None
        peak = peaks.get("bf16_tflops_sustained") or peaks.get("bf16_tflops")
        clocks = clk.summary()
        launches_per_step = sum(n for _, n in ktimes.values()) // max(1, args.steps)
        fp32 = cfg["dtype"] == "f32"
        w_bytes = sum(t.numel() * t.element_size() for t in w_tensors if hasattr(t, "numel"))
        if fp32:
            roof = {"kernel": "mlp_gemm (fp32 CUDA cores)", "bound": "alu", "peak": fp32_alu_peak(peaks),
                    "peak_note": "fp32 FMA peak: 148 SMs x 128 lanes x 2 FLOP x max SM clock"}
            precision = "fp32 everywhere (CUDA cores)"
        else:
            roof = {"kernel": "mlp_gemm (tcgen05)", "bound": "tensor", "peak": peak,
                    "peak_note": "%s sustained cuBLAS bf16" % peak_src}
            precision = ("bf16 inputs, weights and outputs; fp16 tensor-core operands and intermediates; "
                         "fp32 accumulation and LayerNorm statistics")
        roof.update({"achieved": achieved, "unit": "TFLOP/s", "frac": (achieved / roof["peak"]) if achieved else None,
                     "traffic": gemm_traffic() if args.workload == WORKLOAD else None})
        l2 = ("L2 flushed (256 MB write) before every step, outside the timed events" if flush is not None else
              "inputs larger than L2 (X %.0f MB, weights %.2f GB per GPU)" % (x_bytes / 1e6, w_bytes / 1e9))
        line = {
            "metric": METRIC, "value": value, "unit": "examples/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32" if fp32 else "f16", "data": "synthetic",
            "config": {"workload": args.workload + ": " + workload_desc(cfg) +
                       (" + prediction head %d->%s->1, sigmoid" % (cfg["n"] * cfg["d"],
                                                                    "->".join(str(v) for v in C.HEAD_HIDDEN))
                        if args.head else ""), "per_gpu_batch": B,
                       "precision": precision,
                       "global_batch": B * world, "seq_len": None, "parallelism": "replicas (batch shards)",
                       "l2": l2, "launch": ("one CUDA graph replay per step" if args.graph else
                                            "eager, one C-ABI call per step") +
                       "; timed with the per-kernel events off, per-kernel times (kernel_ms_per_step, "
                       "roofline.achieved) from a second, profiled pass of the same steps"},
            "tflops_per_gpu": tflops,
            "pct_of_bf16_peak": 100.0 * tflops / peak,
            "peak_source": "%s bf16_tflops_sustained" % peak_src,
            "roofline": roof,
            "kernel_ms_per_step": {k: v[0] / args.steps for k, v in ktimes.items()},
            "clocks": clocks,
            "e2e": {"value": e2e_value, "unit": "examples/s", "h2d_bytes_per_step": step_bytes,
                    "d2h_bytes_per_step": out_bytes, "api": e2e_api},
            "gpu_launches": launches_per_step * args.steps,
        }
        if e2e_sync is not None:
            line["e2e"]["synchronous_call"] = e2e_sync
        if world == 1 and not args.no_cpu_baseline:
            ns = ORACLE_SAMPLE[args.workload]
            v, dt, thr = oracle_sample(cfg, ns)
            line["cpu_baseline"] = {"value": v, "unit": "examples/s", "cores": thr, "kind": "oracle",
                                    "sample": "%d examples through 1 of the %d layers (%.1f s), scaled to the "
                                              "whole stack" % (ns, cfg["layers"], dt)}
        print(json.dumps(line), flush=True)
    api["destroy"]()
    replicas.finish()


if __name__ == "__main__":
    main()
