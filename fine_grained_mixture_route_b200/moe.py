"""Thin ctypes binding of the C ABI in include/moe.h, taking torch tensors.

Argument marshalling only: every step of the layer runs in the library's sm_100a kernels.
torch supplies device memory and the current CUDA stream.  There is no fallback: if the
shared library is missing or the device is not a B200, calls raise.
"""
from __future__ import annotations

import ctypes
import os
from typing import Dict, Optional

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libmoe_b200.so")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, MOE_ERR_INTERNAL = range(6)
MOE_F32, MOE_BF16 = 0, 1
GATE_SOFTMAX_TOPK, GATE_TOPK_SOFTMAX, GATE_SIGMOID_BIAS = 0, 1, 2
FMT_NATIVE, FMT_E4M3, FMT_MXFP8 = 0, 1, 2   # storage of the routed experts' weights (moe_expert_fmt_t)
MX_UP, MX_DOWN = 0, 1                        # block-scaled weight stacks: w1 | w3, w2 (moe_mx_kind_t)

EXPORTED = ("moe_workspace_bytes", "moe_layer_launches", "moe_status_string", "moe_version", "moe_check_device_error", "moe_ws_init",
            "moe_route", "moe_permute", "moe_expert_ffn", "moe_combine", "moe_layer_forward",
            "moe_layer_forward_timed", "moe_permute_no_alloc", "moe_quantize_rows_e4m3", "moe_train_ctx_bytes",
            "moe_backward_workspace_bytes", "moe_layer_forward_train", "moe_layer_backward",
            "moe_layer_backward_timed", "moe_backward_launches", "moe_balance_workspace_bytes",
            "moe_balance_stats", "moe_gather_rows", "moe_segment_ids", "moe_selftest_wait_timeout",
            "moe_mx_scale_bytes", "moe_quantize_weights_mx")
NUM_STAGES = 7
STAGE_NAMES = ("router", "permute", "plan", "gather", "gemm1_swiglu", "gemm2", "combine")
BWD_STAGES = 7
BWD_STAGE_NAMES = ("bwd_prep", "bwd_dh", "bwd_router", "bwd_dx", "bwd_dw2", "bwd_dw13", "bwd_shared_dc_bias")


class MoeShape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in
                ("T", "d", "n_experts", "inter", "top_k", "n_shared", "inter_shared", "has_bias", "dtype",
                 "gate_mode", "routed_fmt")]


class MoeWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "b1", "w3", "b3", "w2", "b2", "s1", "s3", "s2", "sf13", "sf2")]


class MoeGrads(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("w1", "b1", "w3", "b3", "w2", "b2")]


class MoeError(RuntimeError):
    def __init__(self, status: int, where: str, detail: int = 0):
        self.status = status
        self.detail = detail
        msg = _lib().moe_status_string(status).decode()
        super().__init__(f"{where}: {msg}" + (f" (device error bits {detail:#x})" if detail else ""))


_LIB = None


def _lib():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m fine_grained_mixture_route_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        vp, sz, i32p, f32p = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
        sh = ctypes.POINTER(MoeShape)
        wp = ctypes.POINTER(MoeWeights)
        lib.moe_workspace_bytes.argtypes = [sh]
        lib.moe_workspace_bytes.restype = sz
        lib.moe_layer_launches.argtypes = [sh]
        lib.moe_layer_launches.restype = ctypes.c_int32
        lib.moe_status_string.argtypes = [ctypes.c_int]
        lib.moe_status_string.restype = ctypes.c_char_p
        lib.moe_version.argtypes = []
        lib.moe_version.restype = ctypes.c_char_p
        lib.moe_check_device_error.argtypes = [vp, sz, vp, ctypes.POINTER(ctypes.c_uint32)]
        lib.moe_ws_init.argtypes = [vp, sz, vp]
        lib.moe_route.argtypes = [sh, vp, vp, f32p, i32p, f32p, vp, sz, vp]
        lib.moe_permute.argtypes = [sh, i32p, f32p, i32p, i32p, i32p, f32p, i32p, vp, sz, vp]
        lib.moe_expert_ffn.argtypes = [sh, vp, i32p, i32p, f32p, wp, vp, vp, sz, vp]
        lib.moe_combine.argtypes = [sh, vp, wp, vp, i32p, vp, vp, sz, vp]
        lib.moe_layer_forward.argtypes = [sh, vp, vp, f32p, wp, wp, vp, i32p, f32p, i32p, vp, sz, vp]
        lib.moe_layer_forward_timed.argtypes = [sh, vp, vp, f32p, wp, wp, vp, i32p, f32p, i32p, vp, sz, vp,
                                                ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
        lib.moe_quantize_rows_e4m3.argtypes = [vp, i32p, ctypes.c_int64, ctypes.c_int32, ctypes.c_int32, vp, f32p,
                                               vp, sz, vp]
        gp = ctypes.POINTER(MoeGrads)
        lib.moe_train_ctx_bytes.argtypes = [sh]
        lib.moe_train_ctx_bytes.restype = sz
        lib.moe_backward_workspace_bytes.argtypes = [sh]
        lib.moe_backward_workspace_bytes.restype = sz
        lib.moe_layer_forward_train.argtypes = [sh, vp, vp, f32p, wp, wp, vp, vp, sz, vp, sz, vp]
        lib.moe_layer_backward.argtypes = [sh, vp, vp, f32p, wp, wp, vp, vp, sz, vp, f32p, f32p, gp, gp, vp, sz, vp]
        lib.moe_layer_backward_timed.argtypes = [sh, vp, vp, f32p, wp, wp, vp, vp, sz, vp, f32p, f32p, gp, gp, vp, sz,
                                                 vp, ctypes.POINTER(ctypes.c_void_p), ctypes.c_int32]
        lib.moe_balance_workspace_bytes.argtypes = [sh]
        lib.moe_balance_workspace_bytes.restype = sz
        lib.moe_balance_stats.argtypes = [sh, vp, vp, f32p, i32p, ctypes.c_int32, f32p, f32p, f32p, vp, sz, vp]
        lib.moe_gather_rows.argtypes = [vp, i32p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int32, vp, vp, sz, vp]
        lib.moe_segment_ids.argtypes = [i32p, ctypes.c_int32, ctypes.c_int32, ctypes.c_int64, i32p, vp, sz, vp]
        lib.moe_selftest_wait_timeout.argtypes = [ctypes.c_uint64, vp, vp, sz, vp]
        lib.moe_mx_scale_bytes.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        lib.moe_mx_scale_bytes.restype = sz
        lib.moe_quantize_weights_mx.argtypes = [ctypes.c_int32, vp, vp, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                                vp, vp, vp, vp]
        lib.moe_backward_launches.argtypes = [sh]
        lib.moe_backward_launches.restype = ctypes.c_int32
        for n in ("moe_check_device_error", "moe_ws_init", "moe_route", "moe_permute", "moe_expert_ffn",
                  "moe_combine", "moe_layer_forward", "moe_layer_forward_timed", "moe_quantize_rows_e4m3",
                  "moe_layer_forward_train", "moe_layer_backward", "moe_layer_backward_timed", "moe_balance_stats",
                  "moe_gather_rows", "moe_segment_ids", "moe_selftest_wait_timeout", "moe_quantize_weights_mx"):
            getattr(lib, n).restype = ctypes.c_int
        _LIB = lib
    return _LIB


def lib_handle():
    """The loaded ctypes library (for tests that check the exported symbols)."""
    return _lib()


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, where: str):
    if status != MOE_OK:
        raise MoeError(status, where)


def make_shape(T: int, d: int, n_experts: int, inter: int, top_k: int, n_shared: int = 0, inter_shared: int = 0,
               has_bias: bool = True, dtype: torch.dtype = torch.bfloat16, gate_mode: int = GATE_SOFTMAX_TOPK,
               routed_fmt: int = FMT_NATIVE) -> MoeShape:
    return MoeShape(T, d, n_experts, inter, top_k, n_shared, inter_shared if n_shared else 0, int(bool(has_bias)),
                    MOE_BF16 if dtype == torch.bfloat16 else MOE_F32, gate_mode, routed_fmt)


def shape_of(x: torch.Tensor, centroids_or_E, routed: Dict, top_k: int, shared: Optional[Dict] = None,
             gate_mode: int = GATE_SOFTMAX_TOPK) -> MoeShape:
    E = centroids_or_E if isinstance(centroids_or_E, int) else centroids_or_E.shape[0]
    I = routed["w1"].shape[1]
    Ks = 0 if shared is None else shared["w1"].shape[0]
    Is = 0 if shared is None else shared["w1"].shape[1]
    fmt = FMT_NATIVE                                                         # codes from quant.quantize_stack:
    if routed["w1"].dtype == torch.uint8:                                    # block scales (sf13) or per-row ones
        fmt = FMT_MXFP8 if routed.get("sf13") is not None else FMT_E4M3
    return make_shape(x.shape[0], x.shape[1], E, I, top_k, Ks, Is, routed.get("b1") is not None, x.dtype, gate_mode,
                      fmt)


# ----------------------------------------------------------------------------- argument checks
# The C ABI sees only pointers: a tensor of the wrong element type or size would make a kernel read
# or write past its allocation.  Every entry point below checks, before any call, that each tensor
# has the element type the shape implies, is contiguous, holds at least the elements the kernels
# touch, and lives on the layer's CUDA device.
def _layer_dtype(shape: MoeShape) -> torch.dtype:
    return torch.bfloat16 if shape.dtype == MOE_BF16 else torch.float32


def _need(t, name: str, numel: int, dtype: torch.dtype, device: Optional[torch.device]):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}; this layer shape needs {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name} holds {t.numel()} elements; the layer shape needs {numel}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}; the layer runs on {device}")


def _device(x: torch.Tensor) -> torch.device:
    if not isinstance(x, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    return x.device


def _on_cuda(dev: torch.device):
    """Last check of every entry point: there is no CPU path."""
    if dev.type != "cuda":
        raise ValueError(f"the layer runs on a CUDA device (sm_100a); got tensors on {dev}")


def _need_stack(w: Optional[Dict], name: str, shape: MoeShape, shared: bool, device, grads: bool = False):
    """An expert stack (or its gradients, grads=True) in the layout of include/moe.h."""
    if w is None:
        return
    E = shape.n_shared if shared else shape.n_experts
    I = shape.inter_shared if shared else shape.inter
    d, dt = shape.d, _layer_dtype(shape)
    codes = not shared and not grads and shape.routed_fmt in (FMT_E4M3, FMT_MXFP8)
    wdt = torch.uint8 if codes else dt
    for k, n, kdt in (("w1", E * I * d, wdt), ("w3", E * I * d, wdt), ("w2", E * d * I, wdt),
                      ("b1", E * I, dt), ("b3", E * I, dt), ("b2", E * d, dt),
                      ("s1", E * I, torch.float32), ("s3", E * I, torch.float32), ("s2", E * d, torch.float32),
                      ("sf13", mx_scale_bytes(MX_UP, E, I, d), torch.uint8),
                      ("sf2", mx_scale_bytes(MX_DOWN, E, d, I), torch.uint8)):
        if k in w:
            _need(w[k], f"{name}.{k}", n, kdt, device)


def _bias_ptr(router_bias: Optional[torch.Tensor]):
    if router_bias is None:
        return None
    if router_bias.dtype != torch.float32 or not router_bias.is_contiguous():
        raise ValueError("router_bias must be a contiguous float32 tensor [n_experts]")
    return ctypes.c_void_p(router_bias.data_ptr())


def _weights(w: Optional[Dict]):
    if w is None:
        return None
    for k in ("w1", "w3", "w2", "b1", "b3", "b2", "s1", "s3", "s2", "sf13", "sf2"):
        t = w.get(k)
        if t is not None and not t.is_contiguous():
            raise ValueError(f"weight {k} must be contiguous")
    if w["w1"].dtype == torch.uint8:
        if w.get("sf13") is not None:
            for k in ("sf13", "sf2"):
                if w.get(k) is None or w[k].dtype != torch.uint8:
                    raise ValueError(f"block-scaled e4m3 weights need uint8 scale bytes {k}")
        else:
            for k in ("s1", "s3", "s2"):
                if w.get(k) is None or w[k].dtype != torch.float32:
                    raise ValueError(f"e4m3 weights need float32 scales {k}")
    names = ("w1", "b1", "w3", "b3", "w2", "b2", "s1", "s3", "s2", "sf13", "sf2")
    return MoeWeights(*(None if w.get(k) is None else w[k].data_ptr() for k in names))


def workspace_bytes(shape: MoeShape) -> int:
    return int(_lib().moe_workspace_bytes(ctypes.byref(shape)))


def layer_launches(shape: MoeShape) -> int:
    """Kernel launches one layer_forward call makes for this shape."""
    return int(_lib().moe_layer_launches(ctypes.byref(shape)))


def new_workspace(shape: MoeShape, device="cuda") -> torch.Tensor:
    n = workspace_bytes(shape)
    if n == 0:
        raise ValueError("invalid layer shape")
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    _check(_lib().moe_ws_init(_ptr(ws), n, _stream()), "moe_ws_init")
    return ws


def check_device_error(ws: torch.Tensor, stream=None) -> int:
    """Synchronises the stream and raises MoeError if a kernel flagged an error."""
    detail = ctypes.c_uint32(0)
    st = _lib().moe_check_device_error(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(detail))
    if st != MOE_OK:
        raise MoeError(st, "moe_check_device_error", detail.value)
    return 0


def route(shape: MoeShape, x, centroids, ws, idx=None, gate=None, stream=None, router_bias=None):
    T, k = shape.T, shape.top_k
    dev, dt = _device(x), _layer_dtype(shape)
    _need(x, "x", T * shape.d, dt, dev)
    _need(centroids, "centroids", shape.n_experts * shape.d, dt, dev)
    _need(idx, "idx", T * k, torch.int32, dev)
    _need(gate, "gate", T * k, torch.float32, dev)
    _need(router_bias, "router_bias", shape.n_experts, torch.float32, dev)
    _on_cuda(dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=x.device) if idx is None else idx
    gate = torch.empty((T, k), dtype=torch.float32, device=x.device) if gate is None else gate
    _check(_lib().moe_route(ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias), _ptr(idx),
                            _ptr(gate), _ptr(ws), ws.numel(), _stream(stream)), "moe_route")
    return idx, gate


def permute(shape: MoeShape, idx, gate, ws, stream=None):
    S, E = shape.T * shape.top_k, shape.n_experts
    dev = _device(idx)
    _need(idx, "idx", S, torch.int32, dev)
    _need(gate, "gate", S, torch.float32, dev)
    _on_cuda(dev)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    sorted_token = torch.empty(S, dtype=torch.int32, device=dev)
    sorted_gate = torch.empty(S, dtype=torch.float32, device=dev)
    slot_of = torch.empty(S, dtype=torch.int32, device=dev)
    _check(_lib().moe_permute(ctypes.byref(shape), _ptr(idx), _ptr(gate), _ptr(counts), _ptr(offsets),
                              _ptr(sorted_token), _ptr(sorted_gate), _ptr(slot_of), _ptr(ws), ws.numel(),
                              _stream(stream)), "moe_permute")
    return {"counts": counts, "offsets": offsets, "sorted_token": sorted_token, "sorted_gate": sorted_gate,
            "slot_of": slot_of}


def expert_ffn(shape: MoeShape, x, offsets, sorted_token, sorted_gate, routed: Dict, ws, y=None, stream=None):
    S = shape.T * shape.top_k
    dev, dt = _device(x), _layer_dtype(shape)
    _need(x, "x", shape.T * shape.d, dt, dev)
    _need(offsets, "offsets", shape.n_experts + 1, torch.int32, dev)
    _need(sorted_token, "sorted_token", S, torch.int32, dev)
    _need(sorted_gate, "sorted_gate", S, torch.float32, dev)
    _need(y, "y", S * shape.d, dt, dev)
    _need_stack(routed, "routed", shape, False, dev)
    _on_cuda(dev)
    y = torch.empty((S, shape.d), dtype=x.dtype, device=x.device) if y is None else y
    w = _weights(routed)
    _check(_lib().moe_expert_ffn(ctypes.byref(shape), _ptr(x), _ptr(offsets), _ptr(sorted_token), _ptr(sorted_gate),
                                 ctypes.byref(w), _ptr(y), _ptr(ws), ws.numel(), _stream(stream)), "moe_expert_ffn")
    return y


def combine(shape: MoeShape, x, shared: Optional[Dict], y_sorted, slot_of, ws, out=None, stream=None):
    dev, dt = _device(y_sorted), _layer_dtype(shape)
    S = shape.T * shape.top_k
    _need(x if shape.n_shared > 0 else None, "x", shape.T * shape.d, dt, dev)
    _need(y_sorted, "y_sorted", S * shape.d, dt, dev)
    _need(slot_of, "slot_of", S, torch.int32, dev)
    _need(out, "out", shape.T * shape.d, dt, dev)
    _need_stack(shared, "shared", shape, True, dev)
    _on_cuda(dev)
    out = torch.empty((shape.T, shape.d), dtype=y_sorted.dtype, device=y_sorted.device) if out is None else out
    w = _weights(shared)
    _check(_lib().moe_combine(ctypes.byref(shape), _ptr(x), None if w is None else ctypes.byref(w), _ptr(y_sorted),
                              _ptr(slot_of), _ptr(out), _ptr(ws), ws.numel(), _stream(stream)), "moe_combine")
    return out


def _need_layer(shape: MoeShape, x, centroids, routed, shared, out=None, idx=None, gate=None, counts=None,
                router_bias=None):
    dev, dt = _device(x), _layer_dtype(shape)
    T, d, E, k = shape.T, shape.d, shape.n_experts, shape.top_k
    _need(x, "x", T * d, dt, dev)
    _need(centroids, "centroids", E * d, dt, dev)
    _need(out, "out", T * d, dt, dev)
    _need(idx, "idx", T * k, torch.int32, dev)
    _need(gate, "gate", T * k, torch.float32, dev)
    _need(counts, "counts", E, torch.int32, dev)
    _need(router_bias, "router_bias", E, torch.float32, dev)
    _need_stack(routed, "routed", shape, False, dev)
    _need_stack(shared, "shared", shape, True, dev)
    return dev


def layer_forward(shape: MoeShape, x, centroids, routed: Dict, shared: Optional[Dict], ws, out=None,
                  idx=None, gate=None, counts=None, stream=None, router_bias=None):
    """One call of the whole layer; idx / gate / counts are optional output tensors."""
    _on_cuda(_need_layer(shape, x, centroids, routed, shared, out, idx, gate, counts, router_bias))
    out = torch.empty((shape.T, shape.d), dtype=x.dtype, device=x.device) if out is None else out
    rw = _weights(routed)
    sw = _weights(shared)
    _check(_lib().moe_layer_forward(ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias), ctypes.byref(rw),
                                    None if sw is None else ctypes.byref(sw), _ptr(out), _ptr(idx), _ptr(gate),
                                    _ptr(counts), _ptr(ws), ws.numel(), _stream(stream)), "moe_layer_forward")
    return out


def quantize_rows_e4m3(src: torch.Tensor, ws: torch.Tensor, row_of: Optional[torch.Tensor] = None, stream=None):
    """Per-row e4m3 quantisation of bf16 rows (moe_quantize_rows_e4m3): returns (codes uint8
    [n_rows, width], scales fp32 [n_rows]); rows are src[row_of[p]] when row_of is given."""
    if src.dtype != torch.bfloat16 or src.dim() != 2 or not src.is_contiguous():
        raise ValueError("src must be a contiguous bf16 matrix")
    n = src.shape[0] if row_of is None else row_of.shape[0]
    codes = torch.empty((n, src.shape[1]), dtype=torch.uint8, device=src.device)
    scales = torch.empty(n, dtype=torch.float32, device=src.device)
    _check(_lib().moe_quantize_rows_e4m3(_ptr(src), _ptr(row_of), n, src.shape[0], src.shape[1], _ptr(codes),
                                         _ptr(scales), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_quantize_rows_e4m3")
    return codes, scales


def mx_scale_bytes(kind: int, n_experts: int, rows: int, K: int) -> int:
    """Bytes of the tiled scale array of a block-scaled weight stack (moe_mx_scale_bytes)."""
    return int(_lib().moe_mx_scale_bytes(kind, n_experts, rows, K))


def quantize_weights_mx(kind: int, w_a: torch.Tensor, w_b: Optional[torch.Tensor] = None,
                        codes_a: Optional[torch.Tensor] = None, codes_b: Optional[torch.Tensor] = None, stream=None):
    """Block-scaled e4m3 conversion of bf16 weight stacks (moe_quantize_weights_mx).  MX_UP: w_a = w1, w_b = w3
    [E, I, d]; MX_DOWN: w_a = w2 [E, d, I].  Returns (codes_a, codes_b or None, scale bytes [E, bytes / E]);
    codes_a / codes_b may be given (uint8, same shape), e.g. the halves of one [2, E, I, d] buffer."""
    if kind not in (MX_UP, MX_DOWN):
        raise ValueError("kind must be MX_UP or MX_DOWN")
    if (w_b is not None) != (kind == MX_UP):
        raise ValueError("MX_UP takes w1 and w3, MX_DOWN only w2")
    mats = [w_a] if w_b is None else [w_a, w_b]
    for t in mats:
        if t.dtype != torch.bfloat16 or t.dim() != 3 or not t.is_contiguous() or t.device.type != "cuda":
            raise ValueError("weights must be contiguous bf16 [E, rows, K] stacks on a CUDA device")
        if t.shape != w_a.shape or t.device != w_a.device:
            raise ValueError("w1 and w3 must have the same shape and device")
    E, rows, K = w_a.shape
    outs = []
    for t, c in zip(mats, (codes_a, codes_b)):
        if c is None:
            c = torch.empty(t.shape, dtype=torch.uint8, device=t.device)
        _need(c, "codes", t.numel(), torch.uint8, t.device)
        if c.shape != t.shape:
            raise ValueError("codes must have the weights' shape")
        outs.append(c)
    nbytes = mx_scale_bytes(kind, E, rows, K)
    if nbytes == 0:
        raise ValueError("invalid weight stack shape")
    sf = torch.empty((E, nbytes // E), dtype=torch.uint8, device=w_a.device)
    _check(_lib().moe_quantize_weights_mx(kind, _ptr(w_a), _ptr(w_b), E, rows, K, _ptr(outs[0]),
                                          _ptr(outs[1]) if len(outs) > 1 else None, _ptr(sf), _stream(stream)),
           "moe_quantize_weights_mx")
    return outs[0], (outs[1] if len(outs) > 1 else None), sf


def train_ctx_bytes(shape: MoeShape) -> int:
    return int(_lib().moe_train_ctx_bytes(ctypes.byref(shape)))


def backward_workspace_bytes(shape: MoeShape) -> int:
    return int(_lib().moe_backward_workspace_bytes(ctypes.byref(shape)))


def new_train_buffers(shape: MoeShape, device="cuda"):
    """(ctx, backward workspace) for moe_layer_forward_train / moe_layer_backward."""
    nc, nb = train_ctx_bytes(shape), backward_workspace_bytes(shape)
    if nc == 0 or nb == 0:
        raise ValueError("layer shape not supported for training")
    ctx = torch.empty(nc, dtype=torch.uint8, device=device)
    wsb = torch.empty(nb, dtype=torch.uint8, device=device)
    _check(_lib().moe_ws_init(_ptr(wsb), nb, _stream()), "moe_ws_init")
    return ctx, wsb


def layer_forward_train(shape: MoeShape, x, centroids, routed: Dict, shared: Optional[Dict], ws, ctx, out=None,
                        stream=None, router_bias=None):
    """moe_layer_forward plus the training context in ctx."""
    _on_cuda(_need_layer(shape, x, centroids, routed, shared, out, router_bias=router_bias))
    out = torch.empty((shape.T, shape.d), dtype=x.dtype, device=x.device) if out is None else out
    rw, sw = _weights(routed), _weights(shared)
    _check(_lib().moe_layer_forward_train(ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias),
                                          ctypes.byref(rw), None if sw is None else ctypes.byref(sw), _ptr(out),
                                          _ptr(ctx), ctx.numel(), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_layer_forward_train")
    return out


def _grad_stack(w: Dict):
    g = {k: (None if w.get(k) is None else torch.empty_like(w[k])) for k in ("w1", "b1", "w3", "b3", "w2", "b2")}
    return g, MoeGrads(*(None if g[k] is None else g[k].data_ptr() for k in ("w1", "b1", "w3", "b3", "w2", "b2")))


def backward_launches(shape: MoeShape) -> int:
    return int(_lib().moe_backward_launches(ctypes.byref(shape)))


def new_grads(x, centroids, routed: Dict, shared: Optional[Dict], router_bias_grad: bool = False):
    """Output tensors of layer_backward (reusable across calls)."""
    return {"dx": torch.empty_like(x),
            "dcentroids": torch.empty(centroids.shape, dtype=torch.float32, device=x.device),
            "drouter_bias": torch.empty(centroids.shape[0], dtype=torch.float32, device=x.device) if router_bias_grad
            else None,
            "routed": _grad_stack(routed)[0], "shared": _grad_stack(shared)[0] if shared is not None else None}


def _grad_struct(g: Optional[Dict]):
    if g is None:
        return None
    return MoeGrads(*(None if g.get(k) is None else g[k].data_ptr() for k in ("w1", "b1", "w3", "b3", "w2", "b2")))


def layer_backward(shape: MoeShape, x, centroids, routed: Dict, shared: Optional[Dict], dout, ctx, ws_bwd,
                   stream=None, router_bias=None, router_bias_grad: bool = False, grads: Optional[Dict] = None,
                   events=None):
    """moe_layer_backward (moe_layer_backward_timed when `events` holds BWD_STAGES + 1 events):
    returns {dx, dcentroids, drouter_bias (or None), routed: {...}, shared: {...} or None}, written
    into `grads` when given (see new_grads), else into tensors allocated here."""
    dev = _need_layer(shape, x, centroids, routed, shared, router_bias=router_bias)
    _need(dout, "dout", shape.T * shape.d, _layer_dtype(shape), dev)
    g = new_grads(x, centroids, routed, shared, router_bias_grad) if grads is None else grads
    _need(g["dx"], "dx", shape.T * shape.d, _layer_dtype(shape), dev)
    _need(g["dcentroids"], "dcentroids", shape.n_experts * shape.d, torch.float32, dev)
    _need(g.get("drouter_bias"), "drouter_bias", shape.n_experts, torch.float32, dev)
    _need_stack(g["routed"], "grads.routed", shape, False, dev, grads=True)
    _need_stack(g["shared"], "grads.shared", shape, True, dev, grads=True)
    _on_cuda(dev)
    gr_c, gs_c = _grad_struct(g["routed"]), _grad_struct(g["shared"])
    rw, sw = _weights(routed), _weights(shared)
    args = [ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias), ctypes.byref(rw),
            None if sw is None else ctypes.byref(sw), _ptr(dout), _ptr(ctx), ctx.numel(), _ptr(g["dx"]),
            _ptr(g["dcentroids"]), _ptr(g["drouter_bias"]), ctypes.byref(gr_c),
            None if gs_c is None else ctypes.byref(gs_c), _ptr(ws_bwd), ws_bwd.numel(), _stream(stream)]
    if events is None:
        _check(_lib().moe_layer_backward(*args), "moe_layer_backward")
    else:
        arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
        _check(_lib().moe_layer_backward_timed(*args, arr, len(events)), "moe_layer_backward_timed")
    return g


def balance_stats(shape: MoeShape, x, centroids, counts, n_groups: int = 1, router_bias=None, ws=None, stream=None):
    """moe_balance_stats: returns {f, P (fp32 [n_experts]), expert_term, device_term (0-d fp32)}."""
    dev = _device(x)
    _need(x, "x", shape.T * shape.d, _layer_dtype(shape), dev)
    _need(centroids, "centroids", shape.n_experts * shape.d, _layer_dtype(shape), dev)
    _need(counts, "counts", shape.n_experts, torch.int32, dev)
    _need(router_bias, "router_bias", shape.n_experts, torch.float32, dev)
    _on_cuda(dev)
    n = int(_lib().moe_balance_workspace_bytes(ctypes.byref(shape)))
    if n == 0:
        raise ValueError("layer shape not supported for balance statistics")
    if ws is None or ws.numel() < n:
        ws = torch.zeros(n, dtype=torch.uint8, device=x.device)
    E = centroids.shape[0]
    f = torch.empty(E, dtype=torch.float32, device=x.device)
    P = torch.empty(E, dtype=torch.float32, device=x.device)
    terms = torch.empty(2, dtype=torch.float32, device=x.device)
    _check(_lib().moe_balance_stats(ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias),
                                    _ptr(counts), n_groups, _ptr(f), _ptr(P), _ptr(terms), _ptr(ws), ws.numel(),
                                    _stream(stream)), "moe_balance_stats")
    return {"f": f, "P": P, "expert_term": terms[0], "device_term": terms[1]}


def gather_rows(src: torch.Tensor, row_of: torch.Tensor, ws: torch.Tensor, out=None, stream=None):
    """moe_gather_rows: out[p] = src[row_of[p]] (rows = the first dimension; any dtype whose row
    size is a multiple of 4 bytes)."""
    if not src.is_contiguous() or row_of.dtype != torch.int32:
        raise ValueError("src must be contiguous and row_of int32")
    n = row_of.numel()
    out = torch.empty((n,) + tuple(src.shape[1:]), dtype=src.dtype, device=src.device) if out is None else out
    row_bytes = src[0].numel() * src.element_size() if src.shape[0] else src.element_size()
    _check(_lib().moe_gather_rows(_ptr(src), _ptr(row_of), n, src.shape[0], row_bytes, _ptr(out), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_gather_rows")
    return out


def segment_ids(counts: torch.Tensor, modulo: int, n_rows: int, ws: torch.Tensor, out=None, stream=None):
    """ids[r] = (segment holding row r) % modulo for segments of counts[q] consecutive rows
    (moe_segment_ids); int32 [n_rows]."""
    if counts.dtype != torch.int32 or counts.dim() != 1 or not counts.is_contiguous():
        raise ValueError("counts must be a contiguous int32 vector")
    out = torch.empty(n_rows, dtype=torch.int32, device=counts.device) if out is None else out
    _need(out, "ids", n_rows, torch.int32, counts.device)
    _check(_lib().moe_segment_ids(_ptr(counts), counts.numel(), modulo, n_rows, _ptr(out), _ptr(ws), ws.numel(),
                                  _stream(stream)), "moe_segment_ids")
    return out


def selftest_wait_timeout(limit_ns: int, ws: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None):
    """moe_selftest_wait_timeout: runs the bounded-wait give-up path once (error bit 2 in ws);
    out (int64 [2], optional) receives 1 if the wait gave up and the nanoseconds it waited."""
    _need(out, "out", 2, torch.int64, ws.device)
    _check(_lib().moe_selftest_wait_timeout(limit_ns, _ptr(out), _ptr(ws), ws.numel(), _stream(stream)),
           "moe_selftest_wait_timeout")
    return out


def stage_events(stream=None, n_stages: int = NUM_STAGES):
    """n_stages + 1 recorded torch CUDA events whose handles a timed entry point reuses
    (NUM_STAGES for the forward, BWD_STAGES for the backward)."""
    evs = [torch.cuda.Event(enable_timing=True) for _ in range(n_stages + 1)]
    s = torch.cuda.current_stream() if stream is None else stream
    for e in evs:
        e.record(s)            # creates the underlying CUDA event
    return evs


def layer_forward_timed(shape: MoeShape, x, centroids, routed: Dict, shared: Optional[Dict], ws, events,
                        out=None, idx=None, gate=None, counts=None, stream=None, router_bias=None):
    """layer_forward that also records `events` (from stage_events) at the stage boundaries."""
    _on_cuda(_need_layer(shape, x, centroids, routed, shared, out, idx, gate, counts, router_bias))
    out = torch.empty((shape.T, shape.d), dtype=x.dtype, device=x.device) if out is None else out
    rw = _weights(routed)
    sw = _weights(shared)
    arr = (ctypes.c_void_p * len(events))(*[e.cuda_event for e in events])
    _check(_lib().moe_layer_forward_timed(ctypes.byref(shape), _ptr(x), _ptr(centroids), _bias_ptr(router_bias),
                                          ctypes.byref(rw),
                                          None if sw is None else ctypes.byref(sw), _ptr(out), _ptr(idx), _ptr(gate),
                                          _ptr(counts), _ptr(ws), ws.numel(), _stream(stream), arr, len(events)),
           "moe_layer_forward_timed")
    return out


class MoELayer:
    """Convenience holder: the layer's device tensors, its shape and one workspace."""

    def __init__(self, centroids: torch.Tensor, routed: Dict, shared: Optional[Dict], top_k: int, max_tokens: int,
                 gate_mode: int = GATE_SOFTMAX_TOPK, router_bias: Optional[torch.Tensor] = None):
        self.centroids, self.routed, self.shared, self.top_k = centroids, routed, shared, top_k
        self.max_tokens, self.gate_mode, self.router_bias = max_tokens, gate_mode, router_bias
        dummy = torch.empty((max_tokens, centroids.shape[1]), dtype=centroids.dtype, device="meta")
        self.shape_max = shape_of(dummy, centroids, routed, top_k, shared, gate_mode)
        self.ws = new_workspace(self.shape_max, centroids.device)

    def __call__(self, x: torch.Tensor, out=None, idx=None, gate=None, counts=None, stream=None):
        if x.shape[0] > self.max_tokens:
            raise ValueError("more tokens than the workspace was sized for")
        shape = shape_of(x, self.centroids, self.routed, self.top_k, self.shared, self.gate_mode)
        return layer_forward(shape, x, self.centroids, self.routed, self.shared, self.ws, out, idx, gate, counts,
                             stream, router_bias=self.router_bias)


class HostPipeline:
    """The layer over batches that live in pinned host memory, with the copies overlapped.

    Batch i is copied host-to-device on one stream, the layer runs on a second, and the result
    is copied device-to-host on a third; the copy-in of batch i+1 and the copy-out of batch
    i-1 run while batch i is computed.  Two device buffers for input and output alternate, so
    memory use is fixed.  Every batch still crosses PCIe both ways.
    """

    def __init__(self, shape: MoeShape, centroids, routed: Dict, shared: Optional[Dict], ws, device=None,
                 router_bias=None):
        self.shape, self.centroids, self.routed, self.shared, self.ws = shape, centroids, routed, shared, ws
        self.router_bias = router_bias
        dev = centroids.device if device is None else device
        T, d = shape.T, shape.d
        self.xd = [torch.empty((T, d), dtype=centroids.dtype, device=dev) for _ in range(2)]
        self.od = [torch.empty((T, d), dtype=centroids.dtype, device=dev) for _ in range(2)]
        self.s_in, self.s_comp, self.s_out = (torch.cuda.Stream(dev) for _ in range(3))
        self.in_done = [torch.cuda.Event() for _ in range(2)]
        self.comp_done = [torch.cuda.Event() for _ in range(2)]
        self.out_done = [torch.cuda.Event() for _ in range(2)]
        for e in self.comp_done + self.out_done:
            e.record(torch.cuda.current_stream(dev))

    def run(self, x_host, out_host, start_event=None, stop_event=None):
        """x_host / out_host: equal-length lists of pinned CPU tensors [T, d].  Optional
        timing events are recorded before the first copy-in and after the last copy-out."""
        if start_event is not None:
            start_event.record(self.s_in)
            self.s_comp.wait_event(start_event)
            self.s_out.wait_event(start_event)
        for i, (xh, oh) in enumerate(zip(x_host, out_host)):
            b = i & 1
            with torch.cuda.stream(self.s_in):
                self.s_in.wait_event(self.comp_done[b])          # layer of batch i-2 has read xd[b]
                self.xd[b].copy_(xh, non_blocking=True)
                self.in_done[b].record(self.s_in)
            with torch.cuda.stream(self.s_comp):
                self.s_comp.wait_event(self.in_done[b])
                self.s_comp.wait_event(self.out_done[b])         # copy-out of batch i-2 has read od[b]
                layer_forward(self.shape, self.xd[b], self.centroids, self.routed, self.shared, self.ws,
                              out=self.od[b], stream=self.s_comp, router_bias=self.router_bias)
                self.comp_done[b].record(self.s_comp)
            with torch.cuda.stream(self.s_out):
                self.s_out.wait_event(self.comp_done[b])
                oh.copy_(self.od[b], non_blocking=True)
                self.out_done[b].record(self.s_out)
        if stop_event is not None:
            self.s_in.wait_event(self.out_done[(len(x_host) - 1) & 1])
            self.s_out.wait_event(self.in_done[(len(x_host) - 1) & 1])
            stop_event.record(self.s_out)
        return out_host
