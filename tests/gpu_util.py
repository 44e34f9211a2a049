"""Helpers shared by the GPU parity tests: host inputs from the generator copied to
the device, device outputs read back as float64, and the tolerance check."""
import numpy as np
import torch

import synth


def host_normal(shape, tid, std=1.0, mean=0.0, dtype="bf16", seed=11):
    """Generator values on the host: bf16 (uint16 bit patterns), f32, or f16 (the
    generator's fp32 values rounded to fp16 by numpy, nearest-even)."""
    if dtype == "f16":
        arr = np.empty(shape, dtype=np.float32)
        synth.fill_normal_host(arr, seed, tid, mean, std)
        return arr.astype(np.float16)
    arr = np.empty(shape, dtype=np.uint16 if dtype == "bf16" else np.float32)
    synth.fill_normal_host(arr, seed, tid, mean, std)
    return arr


def to_dev(arr, device="cuda"):
    if arr.dtype == np.uint16:
        return torch.from_numpy(arr.view(np.int16).copy()).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(arr)).to(device)


def torch_dtype(dt):
    return {"bf16": torch.bfloat16, "f16": torch.float16, "f32": torch.float32}[dt]


def f64(arr):
    if isinstance(arr, torch.Tensor):
        return arr.detach().float().cpu().numpy().astype(np.float64)
    if arr.dtype == np.uint16:
        return synth.bf16_bits_to_f64(arr).reshape(arr.shape)
    return arr.astype(np.float64)


def oracle_weight(arr):
    """A weight in a storage type the oracle reads (bf16 bits or float32; f16 values
    are exactly representable in float32)."""
    return arr.astype(np.float32) if arr.dtype == np.float16 else arr


def max_scaled_err(got, ref):
    """max |got - ref| / (1 + |ref|), the parity metric of the stack."""
    return float(np.max(np.abs(got - ref) / (1.0 + np.abs(ref))))
