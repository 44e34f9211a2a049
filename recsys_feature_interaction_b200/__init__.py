"""Python binding of the Wukong interaction-stack C ABI (include/wukong.h).

Argument marshalling only: every function here forwards to the entry point of the
same name in ``_lib/libwukong.so`` and raises :class:`WkError` on a non-OK
status. Every step of the forward runs in that library's CUDA kernels; there is
no Python or CPU implementation behind these names, and every one of them
raises ImportError when the library is missing (build it with
``recsys_feature_interaction_b200.build.build()``).

Tensors are passed as torch tensors (device tensors for the device entry points,
host tensors or numpy arrays for ``wk_stack_forward_host``) or as raw integer
addresses. Streams are torch.cuda.Stream objects, raw cudaStream_t integers, or
None (the current torch stream of the tensor's device).
"""
import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "_lib", "libwukong.so")

WK_OK, WK_ERR_INVALID_ARG, WK_ERR_UNSUPPORTED, WK_ERR_OOM, WK_ERR_CUDA, WK_ERR_TIMEOUT, WK_ERR_DEVICE, WK_ERR_NONFINITE = range(8)
WK_F32, WK_BF16, WK_F16 = 0, 1, 2
(WK_KERNEL_FM_LN, WK_KERNEL_MLP_GEMM, WK_KERNEL_LCB, WK_KERNEL_RES_LN, WK_KERNEL_CONVERT, WK_KERNEL_MOE_GATE,
 WK_KERNEL_MOE_COMBINE, WK_KERNEL_HEAD, WK_KERNEL_WHALE_ATTN, WK_KERNEL_WHALE_FFN, WK_KERNEL_BW_CONTRACT,
 WK_KERNEL_BW_ROWS, WK_KERNEL_FRONT, WK_KERNEL_COUNT) = range(14)
KERNEL_NAMES = ("fm_ln", "mlp_gemm", "lcb", "res_ln", "convert", "moe_gate", "moe_combine", "head", "whale_attn",
                "whale_ffn", "bw_contract", "bw_rows", "front")
WK_MOE_MAX_EXPERTS = 8


class WkError(RuntimeError):
    def __init__(self, status, where):
        self.status = status
        super().__init__("%s: %s (status %d)" % (where, wk_status_string(status), status))


class WkStackConfig(ctypes.Structure):
    _fields_ = [("num_layers", ctypes.c_int32), ("n", ctypes.c_int32), ("d", ctypes.c_int32),
                ("k", ctypes.c_int32), ("n_f", ctypes.c_int32), ("n_l", ctypes.c_int32),
                ("mlp_num_linear", ctypes.c_int32), ("mlp_hidden", ctypes.POINTER(ctypes.c_int32)),
                ("dtype", ctypes.c_int), ("ln_eps", ctypes.c_float), ("max_batch", ctypes.c_int64),
                ("operand_dtype", ctypes.c_int)]


class WkLayerWeights(ctypes.Structure):
    _fields_ = [("Y", ctypes.c_void_p), ("W", ctypes.POINTER(ctypes.c_void_p)),
                ("b", ctypes.POINTER(ctypes.c_void_p)), ("fmb_ln_gamma", ctypes.c_void_p),
                ("fmb_ln_beta", ctypes.c_void_p), ("W_L", ctypes.c_void_p), ("out_ln_gamma", ctypes.c_void_p),
                ("out_ln_beta", ctypes.c_void_p)]


class WkMoeGate(ctypes.Structure):
    _fields_ = [("W_g", ctypes.c_void_p), ("b_g", ctypes.c_void_p)]


class WkLayerGrads(ctypes.Structure):
    _fields_ = [("Y", ctypes.c_void_p), ("W", ctypes.POINTER(ctypes.c_void_p)),
                ("b", ctypes.POINTER(ctypes.c_void_p)), ("fmb_ln_gamma", ctypes.c_void_p),
                ("fmb_ln_beta", ctypes.c_void_p), ("W_L", ctypes.c_void_p), ("out_ln_gamma", ctypes.c_void_p),
                ("out_ln_beta", ctypes.c_void_p)]


class WkWhaleConfig(ctypes.Structure):
    _fields_ = [("n", ctypes.c_int32), ("d", ctypes.c_int32), ("L", ctypes.c_int32), ("h", ctypes.c_int32),
                ("dtype", ctypes.c_int), ("ln_eps", ctypes.c_float), ("max_batch", ctypes.c_int64)]


class WkWhaleWeights(ctypes.Structure):
    _fields_ = [("W_F", ctypes.c_void_p), ("b_F", ctypes.c_void_p), ("ln_gamma", ctypes.c_void_p),
                ("ln_beta", ctypes.c_void_p), ("W_up", ctypes.c_void_p), ("W_down", ctypes.c_void_p)]


_lib = None


def lib():
    """The loaded libwukong.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libwukong.so is missing at %s; build it with "
                              "recsys_feature_interaction_b200.build.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i32, i64, ci, cf = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_int, ctypes.c_float
        sig = {
            "wk_stack_create": [ctypes.POINTER(WkStackConfig), ctypes.POINTER(WkLayerWeights), ctypes.POINTER(vp)],
            "wk_stack_forward": [vp, vp, vp, i64, vp],
            "wk_stack_forward_host": [vp, vp, vp, i64, vp],
            "wk_stack_forward_host_async": [vp, vp, vp, i64, vp, ctypes.POINTER(i64)],
            "wk_stack_host_wait": [vp, i64],
            "wk_stack_sync_status": [vp, vp],
            "wk_stack_set_profiling": [vp, ci],
            "wk_stack_kernel_times": [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)],
            "wk_fm_ln": [vp, vp, vp, vp, vp, i64, i32, i32, i32, ci, cf, vp],
            "wk_mlp_linear": [vp, vp, vp, vp, i64, i32, i32, i64, ci, ci, vp],
            "wk_lcb": [vp, vp, vp, i64, i32, i32, i32, i32, ci, vp],
            "wk_res_ln": [vp, vp, vp, vp, vp, i64, i32, ci, cf, vp],
            "wk_device_status": [vp],
            "wk_layer_forward_noalloc": [ctypes.POINTER(WkStackConfig), ctypes.POINTER(WkLayerWeights), vp, vp, i64,
                                         vp],
            "wk_moe_create": [ctypes.POINTER(WkStackConfig), i32, ctypes.POINTER(WkLayerWeights),
                              ctypes.POINTER(WkMoeGate), ctypes.POINTER(vp)],
            "wk_moe_forward": [vp, vp, vp, i64, vp],
            "wk_moe_sync_status": [vp, vp],
            "wk_moe_set_profiling": [vp, ci],
            "wk_moe_kernel_times": [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)],
            "wk_moe_gate_softmax": [vp, vp, vp, vp, i64, i64, i32, ci, vp],
            "wk_moe_combine": [ctypes.POINTER(vp), vp, vp, ctypes.POINTER(vp), ctypes.POINTER(vp), vp, i64, i32, i32,
                               i32, ci, cf, vp],
            "wk_stack_backward": [vp, vp, vp, vp, ctypes.POINTER(WkLayerGrads), i64, vp],
            "wk_stack_backward_events": [vp, vp, vp, vp, ctypes.POINTER(WkLayerGrads), i64, vp,
                                         ctypes.POINTER(vp)],
            "wk_whale_create": [ctypes.POINTER(WkWhaleConfig), ctypes.POINTER(WkWhaleWeights), ctypes.POINTER(vp)],
            "wk_whale_forward": [vp, vp, vp, vp, i64, vp],
            "wk_whale_sync_status": [vp, vp],
            "wk_whale_set_profiling": [vp, ci],
            "wk_whale_kernel_times": [vp, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)],
            "wk_whale_attention": [vp, vp, vp, i64, i32, i32, i32, ci, vp],
            "wk_whale_fusion_ffn": [vp, vp, ctypes.POINTER(WkWhaleWeights), vp, i64, i32, i32, ci, cf, vp],
        }
        for name, args in sig.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = ci
        L.wk_stack_destroy.argtypes = [vp]
        L.wk_stack_destroy.restype = None
        L.wk_moe_destroy.argtypes = [vp]
        L.wk_moe_destroy.restype = None
        L.wk_whale_destroy.argtypes = [vp]
        L.wk_whale_destroy.restype = None
        L.wk_status_string.argtypes = [ci]
        L.wk_status_string.restype = ctypes.c_char_p
        _lib = L
    return _lib


def _addr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if hasattr(t, "data_ptr"):
        return t.data_ptr()
    if hasattr(t, "ctypes"):  # numpy
        return t.ctypes.data
    raise TypeError("expected a tensor, an array or an address, got %r" % type(t))


def _stream(stream, like=None):
    if stream is None:
        import torch
        dev = like.device if (like is not None and hasattr(like, "device") and like.device.type == "cuda") else None
        return torch.cuda.current_stream(dev).cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status, where):
    if status != WK_OK:
        raise WkError(status, where)


def wk_status_string(status):
    return lib().wk_status_string(int(status)).decode()


def _dtype_code(dtype):
    if dtype in (WK_F32, WK_BF16):
        return dtype
    s = str(dtype)
    if "bfloat16" in s or s == "bf16":
        return WK_BF16
    if "float16" in s or s in ("f16", "fp16", "half"):
        return WK_F16
    if "float32" in s or s in ("f32", "fp32"):
        return WK_F32
    raise ValueError("unsupported dtype %r" % (dtype,))


class StackHandle:
    """An opaque wk_stack* plus the Python objects whose memory it borrows."""

    def __init__(self, ptr, cfg, keep):
        self.ptr = ptr
        self.cfg = cfg
        self._keep = keep

    def __del__(self):
        try:
            if self.ptr:
                wk_stack_destroy(self)
        except Exception:
            pass


def _config(cfg, max_batch, dtype, ln_eps, operand_dtype):
    hidden = list(cfg.get("hidden", []))
    m = len(hidden) + 1
    hid = (ctypes.c_int32 * max(1, len(hidden)))(*hidden) if hidden else None
    c = WkStackConfig(int(cfg.get("num_layers", cfg.get("layers", 1))), cfg["n"], cfg["d"], cfg["k"], cfg["n_f"],
                      cfg["n_l"], m, hid, _dtype_code(dtype if dtype is not None else cfg["dtype"]),
                      float(ln_eps), int(max_batch if max_batch is not None else cfg.get("batch", 1)),
                      _dtype_code(operand_dtype) if operand_dtype is not None else WK_F32)
    return c, hid, m


def _layer_array(layers, m, keep):
    arr = (WkLayerWeights * len(layers))()
    for i, w in enumerate(layers):
        Wp = (ctypes.c_void_p * m)(*[_addr(w["W%d" % j]) for j in range(m)])
        bp = (ctypes.c_void_p * m)(*[_addr(w.get("b%d" % j)) for j in range(m)])
        keep += [Wp, bp]
        arr[i] = WkLayerWeights(_addr(w["Y"]), Wp, bp, _addr(w["fmb_gamma"]), _addr(w["fmb_beta"]), _addr(w["W_L"]),
                                _addr(w["out_gamma"]), _addr(w["out_beta"]))
    keep.append(arr)
    return arr


def wk_stack_create(cfg, layers, max_batch=None, dtype=None, ln_eps=0.0, operand_dtype=None):
    """cfg: mapping with num_layers (or layers), n, d, k, n_f, n_l, hidden (the m-1
    hidden widths) and dtype; layers: one mapping per layer with Y, W0..W{m-1},
    b0..b{m-1} (or None), fmb_gamma, fmb_beta, W_L, out_gamma, out_beta."""
    c, hid, m = _config(cfg, max_batch, dtype, ln_eps, operand_dtype)
    keep = [hid, list(layers)]
    arr = _layer_array(layers, m, keep)
    h = ctypes.c_void_p()
    _check(lib().wk_stack_create(ctypes.byref(c), arr, ctypes.byref(h)), "wk_stack_create")
    return StackHandle(h.value, dict(cfg), keep)


def wk_stack_forward(h, X, out, batch=None, stream=None):
    b = X.shape[0] if batch is None else batch
    _check(lib().wk_stack_forward(h.ptr, _addr(X), _addr(out), int(b), _stream(stream, X)), "wk_stack_forward")


def wk_stack_forward_host(h, X_host, out_host, batch=None, stream=None):
    b = X_host.shape[0] if batch is None else batch
    _check(lib().wk_stack_forward_host(h.ptr, _addr(X_host), _addr(out_host), int(b), _stream(stream)),
           "wk_stack_forward_host")


def wk_stack_forward_host_async(h, X_host, out_host, batch=None, stream=None):
    """Enqueues input copy, forward and output copy; returns the call's ticket. X_host and
    out_host (page-locked CPU tensors) must stay alive and untouched until
    wk_stack_host_wait(h, ticket) returns."""
    b = X_host.shape[0] if batch is None else batch
    t = ctypes.c_int64(-1)
    _check(lib().wk_stack_forward_host_async(h.ptr, _addr(X_host), _addr(out_host), int(b), _stream(stream),
                                             ctypes.byref(t)), "wk_stack_forward_host_async")
    return t.value


def wk_stack_host_wait(h, ticket=-1):
    _check(lib().wk_stack_host_wait(h.ptr, int(ticket)), "wk_stack_host_wait")


def wk_stack_sync_status(h, stream=None):
    return lib().wk_stack_sync_status(h.ptr, _stream(stream))


def wk_stack_backward(h, X, dOut, dX, grads, batch=None, stream=None, layer_events=None):
    """grads: one mapping per layer with fp32 device tensors Y, W (list of m), b (list of m),
    fmb_gamma, fmb_beta, W_L, out_gamma, out_beta (overwritten with the gradients).
    layer_events: optional list of torch.cuda.Event, one per layer (None entries skipped);
    event l is recorded on the stream once layer l's gradients are written."""
    b = X.shape[0] if batch is None else batch
    arr = (WkLayerGrads * len(grads))()
    keep = []
    for i, g in enumerate(grads):
        Wp = (ctypes.c_void_p * len(g["W"]))(*[_addr(t) for t in g["W"]])
        bp = (ctypes.c_void_p * len(g["b"]))(*[_addr(t) for t in g["b"]])
        keep += [Wp, bp]
        arr[i] = WkLayerGrads(_addr(g["Y"]), Wp, bp, _addr(g["fmb_gamma"]), _addr(g["fmb_beta"]), _addr(g["W_L"]),
                              _addr(g["out_gamma"]), _addr(g["out_beta"]))
    if layer_events is None:
        _check(lib().wk_stack_backward(h.ptr, _addr(X), _addr(dOut), _addr(dX), arr, int(b), _stream(stream, X)),
               "wk_stack_backward")
        return
    if len(layer_events) != len(grads):
        raise ValueError("one event (or None) per layer")
    import torch

    for e in layer_events:
        if e is not None and not e.cuda_event:  # torch creates the CUDA event at its first record
            e.record(stream if stream is not None else torch.cuda.current_stream(X.device))
    evp = (ctypes.c_void_p * len(layer_events))(*[e.cuda_event if e is not None else None for e in layer_events])
    _check(lib().wk_stack_backward_events(h.ptr, _addr(X), _addr(dOut), _addr(dX), arr, int(b), _stream(stream, X),
                                          evp), "wk_stack_backward_events")


def wk_stack_destroy(h):
    if h.ptr:
        lib().wk_stack_destroy(h.ptr)
        h.ptr = None


def wk_stack_set_profiling(h, enable=True):
    _check(lib().wk_stack_set_profiling(h.ptr, 1 if enable else 0), "wk_stack_set_profiling")


def wk_stack_kernel_times(h):
    """{kernel name: (total_ms, launches)} since the previous call (waits for the events)."""
    ms = (ctypes.c_double * WK_KERNEL_COUNT)()
    n = (ctypes.c_int64 * WK_KERNEL_COUNT)()
    _check(lib().wk_stack_kernel_times(h.ptr, ms, n), "wk_stack_kernel_times")
    return {KERNEL_NAMES[i]: (ms[i], n[i]) for i in range(WK_KERNEL_COUNT)}


def wk_fm_ln(X, Y, gamma, beta, A0, batch, n, d, k, dtype, eps=0.0, stream=None):
    _check(lib().wk_fm_ln(_addr(X), _addr(Y), _addr(gamma), _addr(beta), _addr(A0), int(batch), n, d, k,
                          _dtype_code(dtype), float(eps), _stream(stream, X)), "wk_fm_ln")


def wk_mlp_linear(A, W, bias, C, M, K, N, ldc, relu, dtype, stream=None):
    _check(lib().wk_mlp_linear(_addr(A), _addr(W), _addr(bias), _addr(C), int(M), K, N, int(ldc), int(bool(relu)),
                               _dtype_code(dtype), _stream(stream, A)), "wk_mlp_linear")


def wk_lcb(W_L, X, concat, batch, n, d, n_f, n_l, dtype, stream=None):
    _check(lib().wk_lcb(_addr(W_L), _addr(X), _addr(concat), int(batch), n, d, n_f, n_l, _dtype_code(dtype),
                        _stream(stream, X)), "wk_lcb")


def wk_res_ln(concat, X, gamma, beta, out, rows, d, dtype, eps=0.0, stream=None):
    _check(lib().wk_res_ln(_addr(concat), _addr(X), _addr(gamma), _addr(beta), _addr(out), int(rows), d,
                           _dtype_code(dtype), float(eps), _stream(stream, X)), "wk_res_ln")


def wk_device_status(stream=None):
    return lib().wk_device_status(_stream(stream))


def wk_layer_forward_noalloc(cfg, layer, X, out, batch=None, stream=None, dtype=None, ln_eps=0.0):
    """One Wukong layer with the intermediates in the library's fixed device array
    (no allocation); see include/wukong.h for who needs it and its limits."""
    c, hid, m = _config(cfg, 1, dtype, ln_eps, None)
    keep = [hid]
    arr = _layer_array([layer], m, keep)
    b = X.shape[0] if batch is None else batch
    _check(lib().wk_layer_forward_noalloc(ctypes.byref(c), arr, _addr(X), _addr(out), int(b), _stream(stream, X)),
           "wk_layer_forward_noalloc")


# ------------------------------------------------------------ mixture of experts

class MoeHandle:
    """An opaque wk_moe* plus the Python objects whose memory it borrows."""

    def __init__(self, ptr, cfg, keep):
        self.ptr = ptr
        self.cfg = cfg
        self._keep = keep

    def __del__(self):
        try:
            if self.ptr:
                wk_moe_destroy(self)
        except Exception:
            pass


def wk_moe_create(cfg, experts, gates, max_batch=None, dtype=None, ln_eps=0.0, operand_dtype=None):
    """cfg as for wk_stack_create plus `experts`; experts[l][e]: the layer-weight mapping
    of expert e of MoE layer l; gates[l]: mapping with W_g [E, n*d] and b_g [E] (or None)."""
    c, hid, m = _config(cfg, max_batch, dtype, ln_eps, operand_dtype)
    L = len(experts)
    E = len(experts[0])
    flat = [experts[l][e] for l in range(L) for e in range(E)]
    keep = [hid, flat, list(gates)]
    arr = _layer_array(flat, m, keep)
    garr = (WkMoeGate * L)(*[WkMoeGate(_addr(g["W_g"]), _addr(g.get("b_g"))) for g in gates])
    keep.append(garr)
    h = ctypes.c_void_p()
    _check(lib().wk_moe_create(ctypes.byref(c), E, arr, garr, ctypes.byref(h)), "wk_moe_create")
    return MoeHandle(h.value, dict(cfg), keep)


def wk_moe_forward(h, X, out, batch=None, stream=None):
    b = X.shape[0] if batch is None else batch
    _check(lib().wk_moe_forward(h.ptr, _addr(X), _addr(out), int(b), _stream(stream, X)), "wk_moe_forward")


def wk_moe_sync_status(h, stream=None):
    return lib().wk_moe_sync_status(h.ptr, _stream(stream))


def wk_moe_destroy(h):
    if h.ptr:
        lib().wk_moe_destroy(h.ptr)
        h.ptr = None


def wk_moe_set_profiling(h, enable=True):
    _check(lib().wk_moe_set_profiling(h.ptr, 1 if enable else 0), "wk_moe_set_profiling")


def wk_moe_kernel_times(h):
    """{kernel name: (total_ms, launches)} summed over the experts and the MoE's own kernels."""
    ms = (ctypes.c_double * WK_KERNEL_COUNT)()
    n = (ctypes.c_int64 * WK_KERNEL_COUNT)()
    _check(lib().wk_moe_kernel_times(h.ptr, ms, n), "wk_moe_kernel_times")
    return {KERNEL_NAMES[i]: (ms[i], n[i]) for i in range(WK_KERNEL_COUNT)}


def wk_moe_gate_softmax(X, W_g, b_g, g, batch, nd, num_experts, dtype, stream=None):
    _check(lib().wk_moe_gate_softmax(_addr(X), _addr(W_g), _addr(b_g), _addr(g), int(batch), int(nd),
                                     int(num_experts), _dtype_code(dtype), _stream(stream, X)), "wk_moe_gate_softmax")


def wk_moe_combine(concats, X, g, gammas, betas, out, batch, n, d, dtype, eps=0.0, stream=None):
    E = len(concats)
    cp = (ctypes.c_void_p * E)(*[_addr(c) for c in concats])
    gp = (ctypes.c_void_p * E)(*[_addr(t) for t in gammas])
    bp = (ctypes.c_void_p * E)(*[_addr(t) for t in betas])
    _check(lib().wk_moe_combine(cp, _addr(X), _addr(g), gp, bp, _addr(out), int(batch), int(n), int(d), E,
                                _dtype_code(dtype), float(eps), _stream(stream, X)), "wk_moe_combine")


# ------------------------------------------------------------ prediction head

class WkHead(ctypes.Structure):
    _fields_ = [("num_linear", ctypes.c_int32), ("hidden", ctypes.POINTER(ctypes.c_int32)),
                ("T", ctypes.POINTER(ctypes.c_void_p)), ("c", ctypes.POINTER(ctypes.c_void_p))]


def wk_stack_set_head(h, head):
    """head: mapping with T (list of q weights [out_j, in_j]) and c (list of q biases
    or None entries); in_0 = n*d, out_{q-1} = 1."""
    T = list(head["T"])
    c = list(head.get("c") or [None] * len(T))
    q = len(T)
    hidden = [int(t.shape[0]) for t in T[:-1]]
    hid = (ctypes.c_int32 * max(1, len(hidden)))(*hidden) if hidden else None
    Tp = (ctypes.c_void_p * q)(*[_addr(t) for t in T])
    cp = (ctypes.c_void_p * q)(*[_addr(t) for t in c])
    hs = WkHead(q, hid, Tp, cp)
    L = lib()
    L.wk_stack_set_head.argtypes = [ctypes.c_void_p, ctypes.POINTER(WkHead)]
    L.wk_stack_set_head.restype = ctypes.c_int
    _check(L.wk_stack_set_head(h.ptr, ctypes.byref(hs)), "wk_stack_set_head")
    h._keep.append((T, c, hid, Tp, cp))


def wk_stack_predict(h, X, logit, prob=None, batch=None, stream=None):
    b = X.shape[0] if batch is None else batch
    L = lib()
    L.wk_stack_predict.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.c_int64, ctypes.c_void_p]
    L.wk_stack_predict.restype = ctypes.c_int
    _check(L.wk_stack_predict(h.ptr, _addr(X), _addr(logit), _addr(prob), int(b), _stream(stream, X)),
           "wk_stack_predict")


# ------------------------------------------------------------------ graphs

class GraphHandle:
    """An opaque wk_graph* (one captured forward on fixed buffers) plus what it uses."""

    def __init__(self, ptr, keep):
        self.ptr = ptr
        self._keep = keep

    def __del__(self):
        try:
            if self.ptr:
                wk_graph_destroy(self)
        except Exception:
            pass


def _graph_sig(L):
    vp = ctypes.c_void_p
    for name in ("wk_stack_graph_create", "wk_moe_graph_create"):
        f = getattr(L, name)
        f.argtypes = [vp, vp, vp, ctypes.c_int64, ctypes.POINTER(vp)]
        f.restype = ctypes.c_int
    L.wk_graph_launch.argtypes = [vp, vp]
    L.wk_graph_launch.restype = ctypes.c_int
    L.wk_graph_destroy.argtypes = [vp]
    L.wk_graph_destroy.restype = None


def wk_stack_graph_create(h, X, out, batch=None):
    L = lib()
    _graph_sig(L)
    g = ctypes.c_void_p()
    b = X.shape[0] if batch is None else batch
    _check(L.wk_stack_graph_create(h.ptr, _addr(X), _addr(out), int(b), ctypes.byref(g)), "wk_stack_graph_create")
    return GraphHandle(g.value, [h, X, out])


def wk_moe_graph_create(h, X, out, batch=None):
    L = lib()
    _graph_sig(L)
    g = ctypes.c_void_p()
    b = X.shape[0] if batch is None else batch
    _check(L.wk_moe_graph_create(h.ptr, _addr(X), _addr(out), int(b), ctypes.byref(g)), "wk_moe_graph_create")
    return GraphHandle(g.value, [h, X, out])


def wk_graph_launch(g, stream=None):
    L = lib()
    _graph_sig(L)
    like = g._keep[1] if len(g._keep) > 1 else None
    _check(L.wk_graph_launch(g.ptr, _stream(stream, like)), "wk_graph_launch")


def wk_graph_destroy(g):
    if g.ptr:
        L = lib()
        _graph_sig(L)
        L.wk_graph_destroy(g.ptr)
        g.ptr = None


# ------------------------------------------------------- WHALE attention fusion

class WhaleHandle:
    """An opaque wk_whale* plus the Python objects whose memory it borrows."""

    def __init__(self, ptr, cfg, keep):
        self.ptr = ptr
        self.cfg = cfg
        self._keep = keep

    def __del__(self):
        try:
            if self.ptr:
                wk_whale_destroy(self)
        except Exception:
            pass


def _whale_weights(w):
    return WkWhaleWeights(_addr(w["W_F"]), _addr(w.get("b_F")), _addr(w["ln_gamma"]), _addr(w["ln_beta"]),
                          _addr(w["W_up"]), _addr(w["W_down"]))


def wk_whale_create(cfg, weights, max_batch=None, dtype=None, ln_eps=0.0):
    """cfg: mapping with n, d, L, h and dtype (and batch, the default max_batch);
    weights: mapping with W_F [d, 2d], b_F [d] (or None), ln_gamma, ln_beta [d],
    W_up [h, d], W_down [d, h]."""
    c = WkWhaleConfig(cfg["n"], cfg["d"], cfg["L"], cfg["h"], _dtype_code(dtype if dtype is not None else cfg["dtype"]),
                      float(ln_eps), int(max_batch if max_batch is not None else cfg.get("batch", 1)))
    ww = _whale_weights(weights)
    h = ctypes.c_void_p()
    _check(lib().wk_whale_create(ctypes.byref(c), ctypes.byref(ww), ctypes.byref(h)), "wk_whale_create")
    return WhaleHandle(h.value, dict(cfg), [dict(weights), ww])


def wk_whale_forward(h, Hw, Hs, Hf, batch=None, stream=None):
    b = Hw.shape[0] if batch is None else batch
    _check(lib().wk_whale_forward(h.ptr, _addr(Hw), _addr(Hs), _addr(Hf), int(b), _stream(stream, Hw)),
           "wk_whale_forward")


def wk_whale_sync_status(h, stream=None):
    return lib().wk_whale_sync_status(h.ptr, _stream(stream))


def wk_whale_destroy(h):
    if h.ptr:
        lib().wk_whale_destroy(h.ptr)
        h.ptr = None


def wk_whale_set_profiling(h, enable=True):
    _check(lib().wk_whale_set_profiling(h.ptr, 1 if enable else 0), "wk_whale_set_profiling")


def wk_whale_kernel_times(h):
    """{kernel name: (total_ms, launches)} of the handle's forwards since the last call."""
    ms = (ctypes.c_double * WK_KERNEL_COUNT)()
    n = (ctypes.c_int64 * WK_KERNEL_COUNT)()
    _check(lib().wk_whale_kernel_times(h.ptr, ms, n), "wk_whale_kernel_times")
    return {KERNEL_NAMES[i]: (ms[i], n[i]) for i in range(WK_KERNEL_COUNT)}


def wk_whale_attention(Hw, Hs, A, batch, n, L, d, dtype, stream=None):
    _check(lib().wk_whale_attention(_addr(Hw), _addr(Hs), _addr(A), int(batch), int(n), int(L), int(d),
                                    _dtype_code(dtype), _stream(stream, Hw)), "wk_whale_attention")


def wk_whale_fusion_ffn(Hw, A, weights, Hf, rows, d, h, dtype, eps=0.0, stream=None):
    ww = _whale_weights(weights)
    _check(lib().wk_whale_fusion_ffn(_addr(Hw), _addr(A), ctypes.byref(ww), _addr(Hf), int(rows), int(d), int(h),
                                     _dtype_code(dtype), float(eps), _stream(stream, Hw)), "wk_whale_fusion_ffn")
