"""Seeded synthetic inputs for the Wukong interaction stack.

This module serves both the fp64 oracle and the CUDA path and holds none of the
layer's arithmetic: it maps (seed, tensor id, element index) to a value and
rounds it to the storage type (see ``synth_core.h`` for the definition). The
host fill (``fill_*_host``) and the device fill (``fill_*_dev``) give identical
bits for the same tensor, so the oracle can regenerate on the host exactly what
the GPU was given.

The five workloads and their recipes live in :mod:`synth.configs`.
"""
import ctypes
import os

import numpy as np

from . import build as _build

F32 = 0
BF16 = 1

_host = None
_dev = None


def _host_lib():
    global _host
    if _host is None:
        path = _build.build_host()
        lib = ctypes.CDLL(path)
        u64, i64, dbl, vp, ci = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        lib.synth_fill_normal_host.argtypes = [vp, ci, u64, u64, u64, u64, dbl, dbl, ci]
        lib.synth_fill_x_logscaled_host.argtypes = [vp, ci, u64, u64, u64, u64, u64, i64, i64, ci]
        lib.synth_normal_f64_host.argtypes = [vp, u64, u64, u64, u64]
        lib.synth_log_uniform_f64_host.argtypes = [vp, u64, u64, u64]
        lib.synth_log_f64.argtypes = [dbl]
        lib.synth_log_f64.restype = dbl
        lib.synth_exp_f64.argtypes = [dbl]
        lib.synth_exp_f64.restype = dbl
        lib.synth_cos_sin_2pi_f64.argtypes = [dbl, ctypes.POINTER(dbl), ctypes.POINTER(dbl)]
        lib.synth_f64_to_bf16_bits.argtypes = [dbl]
        lib.synth_f64_to_bf16_bits.restype = ctypes.c_uint16
        for f in ("synth_fill_normal_host", "synth_fill_x_logscaled_host", "synth_normal_f64_host",
                  "synth_log_uniform_f64_host"):
            getattr(lib, f).restype = ci
        _host = lib
    return _host


def _dev_lib():
    global _dev
    if _dev is None:
        path = _build.build_dev()
        lib = ctypes.CDLL(path)
        u64, i64, dbl, vp, ci = ctypes.c_uint64, ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        lib.synth_fill_normal_dev.argtypes = [vp, ci, u64, u64, u64, u64, dbl, dbl, vp]
        lib.synth_fill_x_logscaled_dev.argtypes = [vp, ci, u64, u64, u64, u64, u64, i64, i64, vp]
        lib.synth_fill_normal_dev.restype = ci
        lib.synth_fill_x_logscaled_dev.restype = ci
        _dev = lib
    return _dev


def _host_threads():
    return max(1, min(64, os.cpu_count() or 1))


def _np_dtype_code(arr):
    if arr.dtype == np.float32:
        return F32
    if arr.dtype == np.uint16:  # bf16 stored as its bit pattern
        return BF16
    raise TypeError("host tensors are float32 or uint16 (bf16 bits), got %s" % arr.dtype)


def fill_normal_host(arr, seed, tensor_id, mean=0.0, std=1.0, offset=0):
    """arr.flat[j] = round(mean + std * normal(seed, tensor_id, offset + j))."""
    assert arr.flags["C_CONTIGUOUS"]
    rc = _host_lib().synth_fill_normal_host(arr.ctypes.data, _np_dtype_code(arr), offset, arr.size, seed,
                                            tensor_id, float(mean), float(std), _host_threads())
    if rc:
        raise RuntimeError("synth_fill_normal_host failed")
    return arr


def fill_x_logscaled_host(arr, seed, tensor_id, scale_tensor_id, n_feat, d, offset=0):
    assert arr.flags["C_CONTIGUOUS"]
    rc = _host_lib().synth_fill_x_logscaled_host(arr.ctypes.data, _np_dtype_code(arr), offset, arr.size, seed,
                                                 tensor_id, scale_tensor_id, n_feat, d, _host_threads())
    if rc:
        raise RuntimeError("synth_fill_x_logscaled_host failed")
    return arr


def normal_f64(count, seed, tensor_id, offset=0):
    out = np.empty(count, dtype=np.float64)
    _host_lib().synth_normal_f64_host(out.ctypes.data, offset, count, seed, tensor_id)
    return out


def log_uniform_f64(count, seed, scale_tensor_id):
    out = np.empty(count, dtype=np.float64)
    _host_lib().synth_log_uniform_f64_host(out.ctypes.data, count, seed, scale_tensor_id)
    return out


def _torch_dtype_code(t):
    import torch
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError("device tensors are float32 or bfloat16, got %s" % t.dtype)


def fill_normal_dev(t, seed, tensor_id, mean=0.0, std=1.0, offset=0, stream=None):
    """Device twin of fill_normal_host on a contiguous CUDA tensor."""
    import torch
    assert t.is_cuda and t.is_contiguous()
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    rc = _dev_lib().synth_fill_normal_dev(t.data_ptr(), _torch_dtype_code(t), offset, t.numel(), seed, tensor_id,
                                          float(mean), float(std), ctypes.c_void_p(s.cuda_stream))
    if rc:
        raise RuntimeError("synth_fill_normal_dev failed with code %d" % rc)
    return t


def fill_x_logscaled_dev(t, seed, tensor_id, scale_tensor_id, n_feat, d, offset=0, stream=None):
    import torch
    assert t.is_cuda and t.is_contiguous()
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    rc = _dev_lib().synth_fill_x_logscaled_dev(t.data_ptr(), _torch_dtype_code(t), offset, t.numel(), seed,
                                               tensor_id, scale_tensor_id, n_feat, d,
                                               ctypes.c_void_p(s.cuda_stream))
    if rc:
        raise RuntimeError("synth_fill_x_logscaled_dev failed with code %d" % rc)
    return t


def bf16_bits_to_f64(bits):
    """Exact upcast of bf16 bit patterns (uint16) to float64."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def f64_to_bf16_bits_scalar(x):
    return int(_host_lib().synth_f64_to_bf16_bits(float(x)))
