"""The C ABI boundary without a GPU: the library loads, exports every entry point
that include/wukong.h declares, and rejects invalid arguments before touching a
device."""
import ctypes
import os
import re

import pytest

import recsys_feature_interaction_b200 as wk
from recsys_feature_interaction_b200 import build as wk_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            names += re.findall(r"^WK_API\s+[\w\s\*]+?\b(\w+)\s*\(", text, flags=re.M)
    return names


@pytest.fixture(scope="module")
def L():
    wk_build.build()
    return wk.lib()


def test_exports_every_declared_symbol(L):
    names = _declared_functions()
    assert len(names) >= 13
    for n in names:
        assert hasattr(L, n), n


def test_status_strings(L):
    for s in range(8):
        assert len(wk.wk_status_string(s)) >= 2 and wk.wk_status_string(s) != "unknown status"
    assert wk.wk_status_string(99) == "unknown status"


def _cfg(**kw):
    c = dict(num_layers=1, n=16, d=16, k=4, n_f=8, n_l=8, hidden=[64], dtype="f32", batch=64)
    c.update(kw)
    return c


FAKE = 1 << 20  # aligned, never dereferenced by validation


def _fake_layers(m, count=1):
    layer = {"Y": FAKE, "W_L": FAKE, "fmb_gamma": FAKE, "fmb_beta": FAKE, "out_gamma": FAKE, "out_beta": FAKE}
    for j in range(m):
        layer["W%d" % j] = FAKE
        layer["b%d" % j] = None
    return [layer] * count


@pytest.mark.parametrize("bad,status", [
    (dict(n_f=9), wk.WK_ERR_UNSUPPORTED),          # n_f + n_l != n: no residual projection
    (dict(num_layers=0), wk.WK_ERR_INVALID_ARG),
    (dict(batch=0), wk.WK_ERR_INVALID_ARG),
    (dict(d=12), wk.WK_ERR_UNSUPPORTED),            # d % 8 != 0
    (dict(hidden=[60]), wk.WK_ERR_UNSUPPORTED),     # hidden width % 8 != 0
])
def test_create_rejects_invalid_config_without_gpu(L, bad, status):
    cfg = _cfg(**bad)
    with pytest.raises(wk.WkError) as e:
        wk.wk_stack_create(cfg, _fake_layers(len(cfg["hidden"]) + 1))
    assert e.value.status == status


def test_create_rejects_misaligned_weights(L):
    layers = _fake_layers(2)
    layers = [dict(layers[0], Y=FAKE + 4)]
    with pytest.raises(wk.WkError) as e:
        wk.wk_stack_create(_cfg(), layers)
    assert e.value.status == wk.WK_ERR_INVALID_ARG


def test_create_without_device_reports_cuda_error(L):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    with pytest.raises(wk.WkError) as e:
        wk.wk_stack_create(_cfg(), _fake_layers(2))
    assert e.value.status == wk.WK_ERR_CUDA


def test_null_handle_and_stand_alone_argument_checks(L):
    assert L.wk_stack_forward(None, FAKE, FAKE * 2, 1, None) == wk.WK_ERR_INVALID_ARG
    assert L.wk_stack_sync_status(None, None) == wk.WK_ERR_INVALID_ARG
    t = ctypes.c_int64(7)
    assert L.wk_stack_forward_host_async(None, FAKE, FAKE * 2, 1, None, ctypes.byref(t)) == wk.WK_ERR_INVALID_ARG
    assert t.value == 7  # untouched on an error
    assert L.wk_stack_host_wait(None, -1) == wk.WK_ERR_INVALID_ARG
    assert L.wk_stack_backward(None, FAKE, FAKE, FAKE, None, 8, None) == wk.WK_ERR_INVALID_ARG
    L.wk_stack_destroy(None)
    # misaligned pointers and bad sizes are rejected before any launch
    assert L.wk_mlp_linear(FAKE + 2, FAKE, None, FAKE, 4, 64, 64, 64, 0, 1, None) == wk.WK_ERR_INVALID_ARG
    assert L.wk_mlp_linear(FAKE, FAKE, None, FAKE, 4, 64, 64, 32, 0, 1, None) == wk.WK_ERR_INVALID_ARG
    assert L.wk_res_ln(FAKE, FAKE, FAKE, FAKE, FAKE, -1, 160, 1, ctypes.c_float(0), None) == wk.WK_ERR_INVALID_ARG
    assert L.wk_fm_ln(FAKE, FAKE, FAKE, FAKE, FAKE, 0, 16, 16, 4, 0, ctypes.c_float(0), None) == wk.WK_OK
    assert L.wk_lcb(FAKE, FAKE, FAKE, 3, 16, 16, 8, 8, 7, None) == wk.WK_ERR_UNSUPPORTED


def _moe_status(L, cfg, E, gate_addr=FAKE):
    c, hid, m = wk._config(cfg, None, None, 0.0, None)
    layers = _fake_layers(m, count=max(1, E))
    keep = []
    arr = wk._layer_array(layers, m, keep)
    garr = (wk.WkMoeGate * 1)(wk.WkMoeGate(gate_addr, None))
    h = ctypes.c_void_p()
    return L.wk_moe_create(ctypes.byref(c), E, arr, garr, ctypes.byref(h))


def test_moe_argument_errors_without_a_device(L):
    assert _moe_status(L, _cfg(dtype="bf16"), 0) == wk.WK_ERR_INVALID_ARG
    assert _moe_status(L, _cfg(dtype="bf16"), wk.WK_MOE_MAX_EXPERTS + 1) == wk.WK_ERR_INVALID_ARG
    assert _moe_status(L, _cfg(dtype="f32"), 2) == wk.WK_ERR_UNSUPPORTED
    assert _moe_status(L, _cfg(dtype="bf16"), 2, gate_addr=FAKE + 2) == wk.WK_ERR_INVALID_ARG
    assert _moe_status(L, _cfg(dtype="bf16"), 2, gate_addr=0) == wk.WK_ERR_INVALID_ARG
    with pytest.raises(wk.WkError) as ei:
        wk.wk_moe_gate_softmax(FAKE, FAKE, None, FAKE, 4, 12, 2, "bf16", stream=0)  # nd not a multiple of 8
    assert ei.value.status == wk.WK_ERR_INVALID_ARG
    with pytest.raises(wk.WkError) as ei:
        wk.wk_moe_combine([FAKE] * 9, FAKE, FAKE, [FAKE] * 9, [FAKE] * 9, FAKE, 4, 16, 16, "bf16", stream=0)
    assert ei.value.status == wk.WK_ERR_INVALID_ARG


def test_kernel_kind_count_matches_the_header():
    text = open(os.path.join(ROOT, "include", "wukong.h")).read()
    m = re.search(r"WK_KERNEL_COUNT\s*=\s*(\d+)", text)
    assert m and int(m.group(1)) == wk.WK_KERNEL_COUNT == len(wk.KERNEL_NAMES)


def _whale_status(lib, **kw):
    cfg = dict(n=64, d=128, L=2048, h=512, dtype="bf16", batch=4)
    cfg.update(kw)
    w = {"W_F": FAKE, "b_F": None, "ln_gamma": FAKE, "ln_beta": FAKE, "W_up": FAKE, "W_down": FAKE}
    c = wk.WkWhaleConfig(cfg["n"], cfg["d"], cfg["L"], cfg["h"], wk._dtype_code(cfg["dtype"]), 0.0, cfg["batch"])
    ww = wk._whale_weights(w)
    h = ctypes.c_void_p()
    return lib.wk_whale_create(ctypes.byref(c), ctypes.byref(ww), ctypes.byref(h))


def test_whale_argument_errors_without_a_device(L):
    assert _whale_status(L, d=48) == wk.WK_ERR_UNSUPPORTED
    assert _whale_status(L, d=256) == wk.WK_ERR_UNSUPPORTED
    assert _whale_status(L, h=100) == wk.WK_ERR_UNSUPPORTED
    assert _whale_status(L, dtype="f32") == wk.WK_ERR_UNSUPPORTED
    assert _whale_status(L, n=0) == wk.WK_ERR_INVALID_ARG
    assert _whale_status(L, L=0) == wk.WK_ERR_INVALID_ARG
    assert _whale_status(L, batch=0) == wk.WK_ERR_INVALID_ARG
    c = wk.WkWhaleConfig(64, 128, 2048, 512, wk.WK_BF16, 0.0, 4)
    bad = wk.WkWhaleWeights(FAKE, None, FAKE, FAKE, FAKE + 2, FAKE)  # W_up not 16-byte aligned
    h = ctypes.c_void_p()
    assert L.wk_whale_create(ctypes.byref(c), ctypes.byref(bad), ctypes.byref(h)) == wk.WK_ERR_INVALID_ARG
    assert L.wk_whale_attention(FAKE, FAKE, FAKE, 0, 64, 2048, 128, wk.WK_BF16, None) == wk.WK_OK
    assert L.wk_whale_attention(FAKE, FAKE, FAKE, 2, 64, 2048, 96, wk.WK_BF16, None) == wk.WK_ERR_UNSUPPORTED
    assert L.wk_whale_attention(FAKE, FAKE, FAKE, 2, 64, 0, 128, wk.WK_BF16, None) == wk.WK_ERR_INVALID_ARG
    w = wk.WkWhaleWeights(FAKE, None, FAKE, FAKE, FAKE, FAKE)
    assert L.wk_whale_fusion_ffn(FAKE, FAKE, ctypes.byref(w), FAKE, 5, 128, 96, wk.WK_BF16, ctypes.c_float(0),
                                 None) == wk.WK_ERR_UNSUPPORTED
    assert L.wk_whale_fusion_ffn(FAKE, FAKE, ctypes.byref(w), FAKE, 0, 128, 512, wk.WK_BF16, ctypes.c_float(0),
                                 None) == wk.WK_OK


def _noalloc_status(L, layer, batch):
    c, hid, m = wk._config(_cfg(dtype="bf16"), 1, None, 0.0, None)
    keep = [hid]
    arr = wk._layer_array([layer], m, keep)
    return L.wk_layer_forward_noalloc(ctypes.byref(c), arr, FAKE, FAKE * 4, batch, None)


@pytest.mark.parametrize("key", ["Y", "W0", "b0", "W1", "W_L", "fmb_gamma", "fmb_beta", "out_gamma", "out_beta"])
def test_noalloc_rejects_misaligned_weights_before_any_launch(L, key):
    """wk_layer_forward_noalloc checks every weight, bias and LayerNorm pointer for the
    16-byte alignment its kernels' vector loads and TMA need, on the host, before it looks
    up a device: on a machine without a GPU the answer is still the argument error."""
    layer = dict(_fake_layers(2)[0])
    layer[key] = FAKE + 4
    assert _noalloc_status(L, layer, 8) == wk.WK_ERR_INVALID_ARG


def test_noalloc_rejects_batches_that_would_overflow_the_size_arithmetic(L):
    for batch in (1 << 40, (1 << 62) + 1):
        assert _noalloc_status(L, _fake_layers(2)[0], batch) == wk.WK_ERR_INVALID_ARG
