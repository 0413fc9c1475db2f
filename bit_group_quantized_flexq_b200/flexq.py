"""Python binding of libflexq.so (the C ABI in include/flexq.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  torch supplies device memory and the current CUDA stream.  There is
no fallback: if the library is missing or a call fails, an exception is
raised.
"""

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libflexq.so")

FLEXQ_OK = 0
FLEXQ_ERR_INVALID_ARG = 1
FLEXQ_ERR_UNSUPPORTED = 2
FLEXQ_ERR_MISALIGNED = 3
FLEXQ_ERR_CUDA = 4
FLEXQ_ERR_DEVICE_TIMEOUT = 5

_lib = None
MAX_GROUP_LAYERS = 4
LAYOUT_BYTE_ALIGNED = 0      # the default device form of the packed weights
LAYOUT_4_2 = 1               # the "4+2" bit-plane form


class Layer(ctypes.Structure):
    """flexq_layer_t: one layer of a grouped call."""
    _fields_ = [("N", ctypes.c_int), ("Wq_packed", ctypes.c_void_p),
                ("W_scales", ctypes.c_void_p), ("Y_fp16", ctypes.c_void_p)]


class FlexQError(RuntimeError):
    def __init__(self, status, message):
        super().__init__(message)
        self.status = status


def lib():
    """The loaded library (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"{LIB_PATH} is missing: build it with "
                "`python -m bit_group_quantized_flexq_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        c_int, c_void_p, c_size_t = ctypes.c_int, ctypes.c_void_p, ctypes.c_size_t
        sig = {
            "flexq_status_string": (ctypes.c_char_p, [c_int]),
            "flexq_last_error_message": (ctypes.c_char_p, []),
            "flexq_weight_packed_bytes": (c_size_t, [c_int, c_int, c_int]),
            "flexq_act_scales_ld": (c_size_t, [c_int]),
            "flexq_quantize_weight": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p,
                                              c_void_p, c_void_p]),
            "flexq_quantize_act": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                           c_void_p, c_void_p]),
            "flexq_gemm_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
            "flexq_gemm_w6a6": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
            "flexq_gemm_w6a8": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                        c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                        c_void_p]),
            "flexq_linear_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int]),
            "flexq_linear_w6a6": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "flexq_linear_w6a8": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_size_t, c_void_p]),
            "flexq_gemm_static_scratch": (c_int, [c_int, c_int, c_int, c_int, c_int, c_void_p,
                                                  c_void_p, c_void_p, c_void_p, c_void_p,
                                                  c_void_p]),
            "flexq_debug_check_quantizer": (c_int, [ctypes.POINTER(ctypes.c_ulonglong),
                                                    ctypes.POINTER(ctypes.c_uint)]),
            "flexq_debug_group_partials": (c_int, [c_int, c_int, c_int, c_int, c_void_p,
                                                   c_void_p, c_void_p, c_void_p]),
            "flexq_gemm_plan": (c_int, [c_int, c_int, c_int, c_int,
                                        ctypes.POINTER(c_int), ctypes.POINTER(c_int),
                                        ctypes.POINTER(c_int)]),
            "flexq_debug_force_plan": (c_int, [c_int, c_int]),
            "flexq_linear_launches": (c_int, [c_int, c_int, c_int, c_int]),
            "flexq_debug_export_canonical": (c_int, [c_int, c_int, c_int, c_void_p, c_void_p, c_void_p]),
            "flexq_debug_force_linear_route": (c_int, [c_int]),
            "flexq_set_wait_limit_ns": (c_int, [ctypes.c_uint64]),
            "flexq_debug_inject_stall": (c_int, [c_int]),
            "flexq_get_device_status": (c_int, [c_void_p]),
            "flexq_quantize_weight_layout": (c_int, [c_int, c_int, c_int, c_int, c_void_p,
                                                     c_void_p, c_void_p, c_void_p]),
            "flexq_gemm_layout": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_void_p,
                                          c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                                          c_size_t, c_void_p]),
            "flexq_linear_layout": (c_int, [c_int, c_int, c_int, c_int, c_int, c_int, c_void_p,
                                            c_void_p, c_void_p, c_void_p, c_void_p, c_size_t,
                                            c_void_p]),
            "flexq_gemm_group": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_void_p, c_int,
                                         ctypes.POINTER(Layer), c_void_p, c_size_t, c_void_p]),
            "flexq_linear_group": (c_int, [c_int, c_int, c_int, c_int, c_void_p, c_int,
                                           ctypes.POINTER(Layer), c_void_p, c_size_t,
                                           c_void_p]),
            "flexq_gemm_group_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int,
                                                            ctypes.POINTER(c_int)]),
            "flexq_linear_group_workspace_bytes": (c_size_t, [c_int, c_int, c_int, c_int,
                                                              ctypes.POINTER(c_int)]),
            "flexq_group_plan": (c_int, [c_int, c_int, c_int, c_int, ctypes.POINTER(c_int),
                                         ctypes.POINTER(c_int), ctypes.POINTER(c_int),
                                         ctypes.POINTER(c_int), ctypes.POINTER(c_int)]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status):
    if status != FLEXQ_OK:
        L = lib()
        name = L.flexq_status_string(status).decode()
        detail = L.flexq_last_error_message().decode()
        raise FlexQError(status, f"{name}: {detail}")


def _stream(t=None):
    dev = t.device if t is not None else torch.device("cuda")
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype, shape=None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must live on a CUDA device")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def weight_packed_bytes(N, K, group_size):
    return int(lib().flexq_weight_packed_bytes(N, K, group_size))


def act_scales_ld(M):
    return int(lib().flexq_act_scales_ld(M))


def act_scales_view(xs, M):
    """The [M, G] view of group-major activation scales ([G, ld] storage)."""
    return xs[:, :M].t()


def weight_scales_view(ws):
    """The [N, G] view of group-major weight scales ([G, N] storage)."""
    return ws.t()


def quantize_weight(w, group_size, out=None, layout=LAYOUT_BYTE_ALIGNED):
    """FP16 W [N, K] -> (packed uint8 [3NK/4] in the device form of `layout`,
    FP16 scales stored group-major as a [K/gs, N] tensor)."""
    _need(w, "w", torch.float16)
    N, K = w.shape
    nbytes = weight_packed_bytes(N, K, group_size)
    if nbytes == 0:
        raise FlexQError(FLEXQ_ERR_UNSUPPORTED, f"unsupported weight shape {N}x{K}, gs={group_size}")
    if out is None:
        out = (torch.empty(nbytes, dtype=torch.uint8, device=w.device),
               torch.empty(K // group_size, N, dtype=torch.float16, device=w.device))
    wp, ws = out
    _need(wp, "packed", torch.uint8, (nbytes,))
    _need(ws, "scales", torch.float16, (K // group_size, N))
    if layout == LAYOUT_BYTE_ALIGNED:
        _check(lib().flexq_quantize_weight(N, K, group_size, _ptr(w), _ptr(wp), _ptr(ws),
                                           _stream(w)))
    else:
        _check(lib().flexq_quantize_weight_layout(N, K, group_size, layout, _ptr(w), _ptr(wp),
                                                  _ptr(ws), _stream(w)))
    return wp, ws


def quantize_act(x, group_size, bits, out=None):
    """FP16 X [M, K] -> (int8 codes [M, K], FP16 scales stored group-major as a
    [K/gs, act_scales_ld(M)] tensor; see act_scales_view)."""
    _need(x, "x", torch.float16)
    M, K = x.shape
    ld = act_scales_ld(M)
    if out is None:
        out = (torch.empty(M, K, dtype=torch.int8, device=x.device),
               torch.empty(K // group_size, ld, dtype=torch.float16, device=x.device))
    xq, xs = out
    _need(xq, "codes", torch.int8, (M, K))
    _need(xs, "scales", torch.float16, (K // group_size, ld))
    _check(lib().flexq_quantize_act(M, K, group_size, bits, _ptr(x), _ptr(xq), _ptr(xs), _stream(x)))
    return xq, xs


def gemm_workspace_bytes(M, N, K, group_size):
    return int(lib().flexq_gemm_workspace_bytes(M, N, K, group_size))


# zero-filled split-K workspaces, one growing buffer per device; superseded
# buffers stay alive because captured CUDA graphs may still point at them
_workspaces = {}
_retired = []


def workspace(device, nbytes):
    """A zero-filled device workspace of at least `nbytes` bytes on `device`
    (shared by every call on that device that does not pass its own)."""
    dev = torch.device(device)
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    cur = _workspaces.get(key)
    if cur is None or cur.numel() < nbytes:
        if cur is not None:
            _retired.append(cur)
        cur = torch.zeros(max(nbytes, 1 << 20), dtype=torch.uint8, device=dev)
        _workspaces[key] = cur
    return cur


def reset_workspaces():
    """Zero every workspace handed out by `workspace` (after a device-side
    timeout left split-K counters behind)."""
    for t in list(_workspaces.values()) + _retired:
        t.zero_()


def gemm(xq, xs, wp, ws, N, group_size, act_bits=6, out=None, workspace_buf=None,
         layout=LAYOUT_BYTE_ALIGNED):
    """Y [M, N] FP16 = dequant(xq, xs) . dequant(wp, ws)^T (W6A6 or W6A8).

    workspace_buf: a zero-filled uint8 device tensor of at least
    gemm_workspace_bytes(M, N, K, gs) bytes; by default a per-device shared
    one.  Pass an empty tensor to run without a K split."""
    _need(xq, "xq", torch.int8)
    M, K = xq.shape
    _need(xs, "xs", torch.float16, (K // group_size, act_scales_ld(M)))
    _need(wp, "wp", torch.uint8, (weight_packed_bytes(N, K, group_size),))
    _need(ws, "ws", torch.float16, (K // group_size, N))
    if out is None:
        out = torch.empty(M, N, dtype=torch.float16, device=xq.device)
    _need(out, "out", torch.float16, (M, N))
    if workspace_buf is None:
        need = gemm_workspace_bytes(M, N, K, group_size)
        workspace_buf = workspace(xq.device, need) if need else None
    if workspace_buf is None or workspace_buf.numel() == 0:
        wsp, wsn = ctypes.c_void_p(0), 0
    else:
        _need(workspace_buf, "workspace", torch.uint8)
        wsp, wsn = _ptr(workspace_buf), workspace_buf.numel()
    if layout != LAYOUT_BYTE_ALIGNED:
        _check(lib().flexq_gemm_layout(M, N, K, group_size, act_bits, layout, _ptr(xq), _ptr(xs),
                                       _ptr(wp), _ptr(ws), _ptr(out), wsp, wsn, _stream(xq)))
        return out
    fn = {6: lib().flexq_gemm_w6a6, 8: lib().flexq_gemm_w6a8}[act_bits]
    _check(fn(M, N, K, group_size, _ptr(xq), _ptr(xs), _ptr(wp), _ptr(ws), _ptr(out), wsp, wsn,
              _stream(xq)))
    return out


def linear_workspace_bytes(M, N, K, group_size):
    return int(lib().flexq_linear_workspace_bytes(M, N, K, group_size))


def linear_launches(M, N, K, group_size):
    """1 where linear() quantizes inside the GEMM (one launch), 2 where it runs
    the quantizer and then the GEMM, 0 for unsupported shapes."""
    return int(lib().flexq_linear_launches(M, N, K, group_size))


def force_linear_route(route=0):
    """Test hook: 0 by shape, 1 quantization inside the GEMM wherever the
    plan's token tile is 16 rows, 2 always the separate quantizer."""
    _check(lib().flexq_debug_force_linear_route(route))


def linear(x, wp, ws, N, group_size, act_bits=6, out=None, workspace_buf=None,
           layout=LAYOUT_BYTE_ALIGNED):
    """Y [M, N] FP16 of a quantized linear layer from FP16 activations x
    [M, K]: the activations are quantized to act_bits (6 or 8) by the rule of
    quantize_act, then multiplied with the packed 6-bit weights.  Batches of
    few tokens on short K ranges quantize inside the GEMM (one launch; linear_launches).

    workspace_buf: a zero-filled uint8 device tensor of at least
    linear_workspace_bytes(M, N, K, gs) bytes; by default a per-device shared
    one."""
    _need(x, "x", torch.float16)
    M, K = x.shape
    _need(wp, "wp", torch.uint8, (weight_packed_bytes(N, K, group_size),))
    _need(ws, "ws", torch.float16, (K // group_size, N))
    if out is None:
        out = torch.empty(M, N, dtype=torch.float16, device=x.device)
    _need(out, "out", torch.float16, (M, N))
    if workspace_buf is None:
        need = linear_workspace_bytes(M, N, K, group_size)
        workspace_buf = workspace(x.device, need) if need else None
    if workspace_buf is None or workspace_buf.numel() == 0:
        wsp, wsn = ctypes.c_void_p(0), 0
    else:
        _need(workspace_buf, "workspace", torch.uint8)
        wsp, wsn = _ptr(workspace_buf), workspace_buf.numel()
    if layout != LAYOUT_BYTE_ALIGNED:
        _check(lib().flexq_linear_layout(M, N, K, group_size, act_bits, layout, _ptr(x), _ptr(wp),
                                         _ptr(ws), _ptr(out), wsp, wsn, _stream(x)))
        return out
    fn = {6: lib().flexq_linear_w6a6, 8: lib().flexq_linear_w6a8}[act_bits]
    _check(fn(M, N, K, group_size, _ptr(x), _ptr(wp), _ptr(ws), _ptr(out), wsp, wsn, _stream(x)))
    return out


def gemm_static_scratch(xq, xs, wp, ws, N, group_size, act_bits=6, out=None):
    """The GEMM through flexq_gemm_static_scratch: no workspace argument and
    no device allocation by the library (the split-K scratch is a fixed array
    in device memory shared by all such calls on a device)."""
    _need(xq, "xq", torch.int8)
    M, K = xq.shape
    _need(xs, "xs", torch.float16, (K // group_size, act_scales_ld(M)))
    _need(wp, "wp", torch.uint8, (weight_packed_bytes(N, K, group_size),))
    _need(ws, "ws", torch.float16, (K // group_size, N))
    if out is None:
        out = torch.empty(M, N, dtype=torch.float16, device=xq.device)
    _need(out, "out", torch.float16, (M, N))
    _check(lib().flexq_gemm_static_scratch(M, N, K, group_size, act_bits, _ptr(xq), _ptr(xs),
                                           _ptr(wp), _ptr(ws), _ptr(out), _stream(xq)))
    return out


def debug_check_quantizer():
    """(mismatch count, (x bits, s bits, Q) of the first) of the GPU's fast
    code rule against the IEEE-division rule over all FP16 (x, s > 0) pairs."""
    n = ctypes.c_ulonglong(0)
    first = (ctypes.c_uint * 3)()
    _check(lib().flexq_debug_check_quantizer(ctypes.byref(n), first))
    return n.value, tuple(first)


def debug_group_partials(xq, wp, N, group_size, out=None):
    """int32 [G, M, N] per-group integer partials from the GEMM mainloop."""
    _need(xq, "xq", torch.int8)
    M, K = xq.shape
    G = K // group_size
    if out is None:
        out = torch.empty(G, M, N, dtype=torch.int32, device=xq.device)
    _need(out, "out", torch.int32, (G, M, N))
    _check(lib().flexq_debug_group_partials(M, N, K, group_size, _ptr(xq), _ptr(wp), _ptr(out),
                                            _stream(xq)))
    return out


def export_canonical(wp, N, K, layout=LAYOUT_BYTE_ALIGNED, out=None):
    """The packed weights wp (device form of `layout`) in the canonical 6-bit
    form: uint8 [N, 3K/4], four codes per three bytes, row-major."""
    _need(wp, "packed", torch.uint8, (N * K * 3 // 4,))
    if out is None:
        out = torch.empty(N, K * 3 // 4, dtype=torch.uint8, device=wp.device)
    _need(out, "out", torch.uint8, (N, K * 3 // 4))
    _check(lib().flexq_debug_export_canonical(N, K, layout, _ptr(wp), _ptr(out), _stream(wp)))
    return out


def plan(M, N, K, group_size):
    """(tokens per tile, K split, CTAs) of the GEMM launch for a shape."""
    t, s, c = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().flexq_gemm_plan(M, N, K, group_size, ctypes.byref(t), ctypes.byref(s),
                                 ctypes.byref(c)))
    return t.value, s.value, c.value


def force_plan(tile_tokens=0, k_split=0):
    _check(lib().flexq_debug_force_plan(tile_tokens, k_split))


def set_wait_limit_ns(ns):
    _check(lib().flexq_set_wait_limit_ns(int(ns)))


def inject_stall(enable=True):
    _check(lib().flexq_debug_inject_stall(1 if enable else 0))


def device_status(device=None):
    """Synchronizes the current stream and returns (status, message); clears it."""
    s = ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)
    st = lib().flexq_get_device_status(s)
    msg = lib().flexq_last_error_message().decode()
    if st == FLEXQ_ERR_DEVICE_TIMEOUT:
        reset_workspaces()
    return st, msg


# ------------------------------------------------------------ grouped calls
def _n_array(Ns):
    return (ctypes.c_int * len(Ns))(*Ns)


def group_plan(M, K, group_size, Ns):
    """(tokens per tile, K split, CTAs, launches of linear_group) for layers of
    widths Ns that share their activations."""
    t, s, c, n = ctypes.c_int(), ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    _check(lib().flexq_group_plan(M, K, group_size, len(Ns), _n_array(Ns), ctypes.byref(t),
                                  ctypes.byref(s), ctypes.byref(c), ctypes.byref(n)))
    return t.value, s.value, c.value, n.value


def gemm_group_workspace_bytes(M, K, group_size, Ns):
    return int(lib().flexq_gemm_group_workspace_bytes(M, K, group_size, len(Ns), _n_array(Ns)))


def linear_group_workspace_bytes(M, K, group_size, Ns):
    return int(lib().flexq_linear_group_workspace_bytes(M, K, group_size, len(Ns), _n_array(Ns)))


def _layers(weights, outs, K, group_size, M, device):
    if not 1 <= len(weights) <= MAX_GROUP_LAYERS:
        raise ValueError(f"1..{MAX_GROUP_LAYERS} layers, got {len(weights)}")
    arr = (Layer * len(weights))()
    ys = []
    for i, (wp, ws, N) in enumerate(weights):
        _need(wp, "wp", torch.uint8, (weight_packed_bytes(N, K, group_size),))
        _need(ws, "ws", torch.float16, (K // group_size, N))
        y = outs[i] if outs is not None and outs[i] is not None else \
            torch.empty(M, N, dtype=torch.float16, device=device)
        _need(y, "out", torch.float16, (M, N))
        arr[i] = Layer(N, wp.data_ptr(), ws.data_ptr(), y.data_ptr())
        ys.append(y)
    return arr, ys


def _ws_args(buf, device, need):
    if buf is None:
        buf = workspace(device, need) if need else None
    if buf is None or buf.numel() == 0:
        return ctypes.c_void_p(0), 0
    _need(buf, "workspace", torch.uint8)
    return _ptr(buf), buf.numel()


def gemm_group(xq, xs, weights, group_size, act_bits=6, outs=None, workspace_buf=None):
    """One launch of the group GEMM for layers sharing quantized activations:
    weights = [(wp, ws, N), ...] (1..4 layers); returns their FP16 outputs."""
    _need(xq, "xq", torch.int8)
    M, K = xq.shape
    _need(xs, "xs", torch.float16, (K // group_size, act_scales_ld(M)))
    arr, ys = _layers(weights, outs, K, group_size, M, xq.device)
    wsp, wsn = _ws_args(workspace_buf, xq.device,
                        gemm_group_workspace_bytes(M, K, group_size, [w[2] for w in weights]))
    _check(lib().flexq_gemm_group(M, K, group_size, act_bits, _ptr(xq), _ptr(xs), len(weights),
                                  arr, wsp, wsn, _stream(xq)))
    return ys


def linear_group(x, weights, group_size, act_bits=6, outs=None, workspace_buf=None):
    """Layers [(wp, ws, N), ...] that read the same FP16 activations x [M, K],
    quantized once (act_bits 6 or 8), in one grouped launch (or the
    quantizer and one grouped launch); returns their FP16 outputs."""
    _need(x, "x", torch.float16)
    M, K = x.shape
    arr, ys = _layers(weights, outs, K, group_size, M, x.device)
    wsp, wsn = _ws_args(workspace_buf, x.device,
                        linear_group_workspace_bytes(M, K, group_size, [w[2] for w in weights]))
    _check(lib().flexq_linear_group(M, K, group_size, act_bits, _ptr(x), len(weights), arr, wsp,
                                    wsn, _stream(x)))
    return ys
