"""ButterflyMoE expert forward on B200: a thin Python binding of libbfmoe.so.

Functions carry the C ABI's names (include/bfmoe.h) and take torch tensors
that live on the current CUDA device; torch only provides device memory and
streams.  Every compute step runs in the library's CUDA kernels, and a missing
library raises instead of falling back.

Each expert is W_i = B(phi_i) . W_base . B(theta_i)^T with one shared ternary
base (ButterflyMoE technical summary, gist.science, section 2.1); inference
applies B(theta)^T, the ternary product and B(phi) without forming W_i
(section 2.3).
"""
from __future__ import annotations

import ctypes
import math
from typing import Optional

from . import capi
from .capi import BFMOE_BF16, BFMOE_F32, BfmoeError

__all__ = [
    "BfmoeError", "Layer", "ButterflyMoE", "bfmoe_pack_base", "bfmoe_unpack_base", "bfmoe_router_topk",
    "bfmoe_router_topk_noalloc", "bfmoe_moe_forward", "bfmoe_moe_workspace_size", "bfmoe_prepare_layer",
    "bfmoe_layer_tables_size", "bfmoe_prepare_gate", "bfmoe_gate_parts_size", "bfmoe_backward", "bfmoe_backward_workspace_size",
    "bfmoe_forward", "bfmoe_decode_forward", "bfmoe_materialize_expert", "bfmoe_workspace_size", "bfmoe_router_scratch_size", "bfmoe_check_device_error",
    "bfmoe_launch_count", "bfmoe_profile_enable", "bfmoe_profile_collect", "bfmoe_last_error", "workspace",
]


def _torch():
    import torch
    return torch


def _stream(stream=None):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _need(t, name, dtype=None, cuda=True, contiguous=True):
    if t is None:
        raise ValueError(f"{name} is required")
    if cuda and not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if contiguous and not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.bfloat16:
        return BFMOE_BF16
    if t.dtype == torch.float32:
        return BFMOE_F32
    raise ValueError(f"x must be float32 or bfloat16, got {t.dtype}")


def words_per_row(d: int) -> int:
    return max(1, (d + 15) // 16)


def bfmoe_last_error() -> str:
    return capi.lib().bfmoe_last_error().decode(errors="replace")


def bfmoe_launch_count() -> int:
    return int(capi.lib().bfmoe_launch_count())


def bfmoe_workspace_size(d: int, n_experts: int, T: int, k: int, x_dtype: int) -> int:
    return int(capi.lib().bfmoe_workspace_size(d, n_experts, T, k, x_dtype))


def bfmoe_router_scratch_size(d: int, n_experts: int, T: int, k: int, x_dtype: int) -> int:
    """Scratch bytes the router alone uses (what bfmoe_router_topk_noalloc checks)."""
    return int(capi.lib().bfmoe_router_scratch_size(d, n_experts, T, k, x_dtype))


def workspace(d: int, n_experts: int, T: int, k: int, x_dtype: int, device=None):
    """A device scratch buffer of bfmoe_workspace_size bytes."""
    torch = _torch()
    n = bfmoe_workspace_size(d, n_experts, T, k, x_dtype)
    if n == 0 and T > 0:
        raise ValueError("invalid sizes for a workspace")
    return torch.empty(max(n, 256), dtype=torch.uint8, device=device or "cuda")


def bfmoe_pack_base(w, out=None, stream=None):
    """int8 [d][d] ternary -> uint32 2-bit codes [d][max(1, d/16)] (synchronises)."""
    torch = _torch()
    _need(w, "w", torch.int8)
    d = w.shape[1]
    if w.dim() != 2 or w.shape[0] != d:
        raise ValueError("w must be [d][d]")
    if out is None:
        out = torch.empty((d, words_per_row(d)), dtype=torch.int32, device=w.device)
    capi.check(capi.lib().bfmoe_pack_base(_ptr(w), d, _ptr(out), _stream(stream)))
    return out


def bfmoe_unpack_base(w_packed, d: int, out=None, stream=None):
    """Packed codes -> the exact bf16 matrix [d][d] the tensor-core product uses."""
    torch = _torch()
    _need(w_packed, "w_packed")
    if out is None:
        out = torch.empty((d, d), dtype=torch.bfloat16, device=w_packed.device)
    capi.check(capi.lib().bfmoe_unpack_base(_ptr(w_packed), d, _ptr(out), _stream(stream)))
    return out


def bfmoe_router_topk(x, w_gate, bias, k: int, ws, out=None, stream=None, buckets: bool = True):
    """Returns (idx [T,k] int32, gates [T,k] f32, counts [N], offsets [N+1], rows [T*k]);
    with ``buckets=False`` the last three are None and are not built."""
    torch = _torch()
    _need(x, "x")
    _need(w_gate, "w_gate", torch.float32)
    if bias is not None:
        _need(bias, "bias", torch.float32)
    T, d = x.shape
    N = w_gate.shape[0]
    dev = x.device
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=dev),
               torch.empty((T, k), dtype=torch.float32, device=dev))
        out += (torch.empty((N,), dtype=torch.int32, device=dev),
                torch.empty((N + 1,), dtype=torch.int32, device=dev),
                torch.empty((T * k,), dtype=torch.int32, device=dev)) if buckets else (None, None, None)
    idx, gates, counts, offsets, rows = out
    capi.check(capi.lib().bfmoe_router_topk(
        _ptr(x), _dtype_code(x), T, d, _ptr(w_gate), _ptr(bias), N, k, _ptr(idx), _ptr(gates),
        _ptr(counts), _ptr(offsets), _ptr(rows), _ptr(ws), ws.numel() if ws is not None else 0,
        _stream(stream)))
    return out


def bfmoe_router_topk_noalloc(x, w_gate, bias, k: int, out=None, stream=None):
    """bfmoe_router_topk for callers that cannot allocate device memory at
    call time: no workspace argument, the library's built-in scratch array is
    used instead (see include/bfmoe.h for its size and sharing rules).  The
    outputs must be provided by the caller (``out``) to allocate nothing here;
    without ``out`` this wrapper allocates them with torch for convenience."""
    torch = _torch()
    _need(x, "x")
    _need(w_gate, "w_gate", torch.float32)
    if bias is not None:
        _need(bias, "bias", torch.float32)
    T, d = x.shape
    N = w_gate.shape[0]
    dev = x.device
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=dev),
               torch.empty((T, k), dtype=torch.float32, device=dev),
               torch.empty((N,), dtype=torch.int32, device=dev),
               torch.empty((N + 1,), dtype=torch.int32, device=dev),
               torch.empty((T * k,), dtype=torch.int32, device=dev))
    idx, gates, counts, offsets, rows = out
    capi.check(capi.lib().bfmoe_router_topk_noalloc(
        _ptr(x), _dtype_code(x), T, d, _ptr(w_gate), _ptr(bias), N, k, _ptr(idx), _ptr(gates),
        _ptr(counts), _ptr(offsets), _ptr(rows), _stream(stream)))
    return out


class Layer:
    """Device weights of one ButterflyMoE layer (packed base, alpha, angles)."""

    def __init__(self, w_packed, alpha: float, theta, phi):
        torch = _torch()
        _need(w_packed, "w_packed")
        _need(theta, "theta", torch.float32)
        _need(phi, "phi", torch.float32)
        self.n_experts, L, half = theta.shape
        self.d = 2 * half
        if L != int(round(math.log2(self.d))) or phi.shape != theta.shape:
            raise ValueError("theta and phi must be [N][log2 d][d/2]")
        self.w_packed, self.theta, self.phi = w_packed, theta, phi
        self.alpha = float(alpha)
        self.c = capi.BfmoeLayer(self.d, self.n_experts, w_packed.data_ptr(), ctypes.c_float(alpha),
                                 theta.data_ptr(), phi.data_ptr(), None, None)
        self.tables = None
        self.gate_parts = None

    def prepare(self, stream=None):
        """Build the weight tables once (bfmoe_prepare_layer); later calls with
        this layer read them instead of rebuilding them per call."""
        torch = _torch()
        n = bfmoe_layer_tables_size(self.d, self.n_experts)
        self.tables = torch.empty(max(n, 256), dtype=torch.uint8, device=self.theta.device)
        self.c.tables = None
        bfmoe_prepare_layer(self, self.tables, stream=stream)
        self.c.tables = self.tables.data_ptr()
        return self

    def unprepare(self):
        """Go back to building the tables per call."""
        self.c.tables = None
        self.tables = None
        return self

    def prepare_gate(self, w_gate, stream=None):
        """Split the router weights once (bfmoe_prepare_gate); the combined
        calls with this layer and the same w_gate then skip the split."""
        torch = _torch()
        _need(w_gate, "w_gate", torch.float32)
        N, d = w_gate.shape
        n = int(capi.lib().bfmoe_gate_parts_size(N, d))
        self.gate_parts = torch.empty(max(n, 256), dtype=torch.uint8, device=w_gate.device)
        capi.check(capi.lib().bfmoe_prepare_gate(_ptr(w_gate), N, d, _ptr(self.gate_parts), self.gate_parts.numel(),
                                                _stream(stream)))
        self.c.gate_parts = self.gate_parts.data_ptr()
        return self

    def unprepare_gate(self):
        """Go back to splitting the router weights per call."""
        self.c.gate_parts = None
        self.gate_parts = None
        return self

    @classmethod
    def from_host(cls, w_base, alpha, theta, phi, device="cuda", stream=None):
        """Pack an int8 ternary base and upload float32 angles."""
        torch = _torch()
        w = torch.as_tensor(w_base, dtype=torch.int8).to(device).contiguous()
        packed = bfmoe_pack_base(w, stream=stream)
        th = torch.as_tensor(theta, dtype=torch.float32).to(device).contiguous()
        ph = torch.as_tensor(phi, dtype=torch.float32).to(device).contiguous()
        return cls(packed, float(alpha), th, ph)


def bfmoe_gate_parts_size(n_experts: int, d: int) -> int:
    return int(capi.lib().bfmoe_gate_parts_size(n_experts, d))


def bfmoe_prepare_gate(w_gate, parts, stream=None):
    """Write the exact bf16 split of w_gate [N][d] into parts (device bytes)."""
    N, d = w_gate.shape
    capi.check(capi.lib().bfmoe_prepare_gate(_ptr(w_gate), N, d, _ptr(parts), parts.numel(), _stream(stream)))
    return parts


def bfmoe_layer_tables_size(d: int, n_experts: int) -> int:
    return int(capi.lib().bfmoe_layer_tables_size(d, n_experts))


def bfmoe_prepare_layer(layer: "Layer", tables, stream=None):
    """Write the layer's weight tables (cos/sin of the angles, bf16 base) into
    ``tables`` (a device byte tensor of bfmoe_layer_tables_size bytes)."""
    _need(tables, "tables")
    capi.check(capi.lib().bfmoe_prepare_layer(ctypes.byref(layer.c), _ptr(tables), tables.numel(), _stream(stream)))
    return tables


def bfmoe_forward(layer: Layer, x, k: int, idx, gates, offsets, rows, ws, y=None, stream=None):
    """y [T][d] (dtype of x) = sum_j g_j B(phi) (alpha W_base (B(theta)^T x))."""
    torch = _torch()
    _need(x, "x")
    T, d = x.shape
    if d != layer.d:
        raise ValueError(f"x has width {d}, layer has d={layer.d}")
    if y is None:
        y = torch.empty_like(x)
    capi.check(capi.lib().bfmoe_forward(
        ctypes.byref(layer.c), _ptr(x), _dtype_code(x), T, k, _ptr(idx), _ptr(gates), _ptr(offsets),
        _ptr(rows), _ptr(y), _ptr(ws), ws.numel() if ws is not None else 0, _stream(stream)))
    return y


def bfmoe_decode_forward(layer: Layer, x, k: int, idx, gates, y=None, stream=None):
    """Add-only small-batch forward: y [T][d] (dtype of x) from the routing
    idx / gates, the ternary product done by signed sums, float32 inside."""
    torch = _torch()
    _need(x, "x")
    T, d = x.shape
    if d != layer.d:
        raise ValueError(f"x has width {d}, layer has d={layer.d}")
    _need(idx, "idx", torch.int32)
    _need(gates, "gates", torch.float32)
    if y is None:
        y = torch.empty_like(x)
    capi.check(capi.lib().bfmoe_decode_forward(
        ctypes.byref(layer.c), _ptr(x), _dtype_code(x), T, k, _ptr(idx), _ptr(gates), _ptr(y), _stream(stream)))
    return y


def bfmoe_backward_workspace_size(d: int, n_experts: int, T: int, k: int) -> int:
    return int(capi.lib().bfmoe_backward_workspace_size(d, n_experts, T, k))


def bfmoe_backward(layer: Layer, x, k: int, w_gate, routing, gy, bias_grad: bool = True, ws=None, stream=None):
    """Gradients of the layer for dL/dy = gy (float32 [T][d]), with the
    forward's routing (idx, gates, counts, offsets, rows).  Returns a dict of
    float32 tensors dx, dtheta, dphi, dw_base, dalpha, dw_gate and dbias
    (None when bias_grad is False)."""
    torch = _torch()
    _need(x, "x")
    _need(w_gate, "w_gate", torch.float32)
    _need(gy, "gy", torch.float32)
    T, d = x.shape
    if d != layer.d or tuple(gy.shape) != (T, d):
        raise ValueError("x and gy must be [T][d] with the layer's d")
    N = layer.n_experts
    idx, gates, _counts, offsets, rows = routing
    dev = x.device
    if ws is None:
        n = bfmoe_backward_workspace_size(d, N, T, k)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    f = dict(dtype=torch.float32, device=dev)
    out = {"dx": torch.empty((T, d), **f), "dtheta": torch.empty_like(layer.theta),
           "dphi": torch.empty_like(layer.phi), "dw_base": torch.empty((d, d), **f),
           "dalpha": torch.empty((1,), **f), "dw_gate": torch.empty((N, d), **f),
           "dbias": torch.empty((N,), **f) if bias_grad else None}
    capi.check(capi.lib().bfmoe_backward(
        ctypes.byref(layer.c), _ptr(x), _dtype_code(x), T, k, _ptr(w_gate), _ptr(idx), _ptr(gates), _ptr(offsets),
        _ptr(rows), _ptr(gy), _ptr(out["dx"]), _ptr(out["dtheta"]), _ptr(out["dphi"]), _ptr(out["dw_base"]),
        _ptr(out["dalpha"]), _ptr(out["dw_gate"]), _ptr(out["dbias"]), _ptr(ws), ws.numel(), _stream(stream)))
    return out


def bfmoe_moe_workspace_size(d: int, n_experts: int, T: int, k: int, x_dtype: int) -> int:
    return int(capi.lib().bfmoe_moe_workspace_size(d, n_experts, T, k, x_dtype))


def bfmoe_moe_forward(layer: Layer, x, w_gate, bias, k: int, ws, routing=None, y=None, stream=None):
    """Router + forward in one call (weight-only work overlaps the router on a
    side stream).  Returns (y, (idx, gates, counts, offsets, rows))."""
    torch = _torch()
    _need(x, "x")
    _need(w_gate, "w_gate", torch.float32)
    if bias is not None:
        _need(bias, "bias", torch.float32)
    T, d = x.shape
    if d != layer.d:
        raise ValueError(f"x has width {d}, layer has d={layer.d}")
    N = layer.n_experts
    dev = x.device
    if routing is None:
        routing = (torch.empty((T, k), dtype=torch.int32, device=dev),
                   torch.empty((T, k), dtype=torch.float32, device=dev),
                   torch.empty((N,), dtype=torch.int32, device=dev),
                   torch.empty((N + 1,), dtype=torch.int32, device=dev),
                   torch.empty((T * k,), dtype=torch.int32, device=dev))
    if y is None:
        y = torch.empty_like(x)
    idx, gates, counts, offsets, rows = routing
    capi.check(capi.lib().bfmoe_moe_forward(
        ctypes.byref(layer.c), _ptr(x), _dtype_code(x), T, _ptr(w_gate), _ptr(bias), k, _ptr(idx), _ptr(gates),
        _ptr(counts), _ptr(offsets), _ptr(rows), _ptr(y), _ptr(ws), ws.numel() if ws is not None else 0,
        _stream(stream)))
    return y, routing


def bfmoe_moe_host_workspace_size(d: int, n_experts: int, T: int, k: int, x_dtype: int, chunk: int = 0) -> int:
    return int(capi.lib().bfmoe_moe_host_workspace_size(d, n_experts, T, k, x_dtype, chunk))


def bfmoe_moe_forward_host(layer: Layer, x_host, w_gate, bias, k: int, y_host, ws, chunk: int = 0, stream=None):
    """Router + forward from and to host memory (pinned CPU tensors), the
    copies overlapped with the work in chunks of ``chunk`` tokens.  ``y_host``
    is complete once ``stream`` has been synchronised.  Returns y_host."""
    torch = _torch()
    for t, name in ((x_host, "x_host"), (y_host, "y_host")):
        if t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor")
    if y_host.shape != x_host.shape or y_host.dtype != x_host.dtype:
        raise ValueError("y_host must match x_host in shape and dtype")
    _need(w_gate, "w_gate", torch.float32)
    if bias is not None:
        _need(bias, "bias", torch.float32)
    T, d = x_host.shape
    if d != layer.d:
        raise ValueError(f"x has width {d}, layer has d={layer.d}")
    capi.check(capi.lib().bfmoe_moe_forward_host(
        ctypes.byref(layer.c), ctypes.c_void_p(x_host.data_ptr()), _dtype_code(x_host), T, _ptr(w_gate), _ptr(bias),
        k, ctypes.c_void_p(y_host.data_ptr()), chunk, _ptr(ws), ws.numel() if ws is not None else 0,
        _stream(stream)))
    return y_host


def bfmoe_materialize_expert(layer: Layer, e: int, out=None, stream=None):
    """alpha * B(phi_e) . W_base . B(theta_e)^T as float32 [d][d] (checking aid)."""
    torch = _torch()
    if out is None:
        out = torch.empty((layer.d, layer.d), dtype=torch.float32, device=layer.theta.device)
    capi.check(capi.lib().bfmoe_materialize_expert(ctypes.byref(layer.c), e, _ptr(out), _stream(stream)))
    return out


def bfmoe_check_device_error(stream=None) -> None:
    capi.check(capi.lib().bfmoe_check_device_error(_stream(stream)))


def bfmoe_profile_enable(on: bool = True) -> None:
    capi.check(capi.lib().bfmoe_profile_enable(1 if on else 0))


def bfmoe_profile_collect():
    """{kernel name: (launches, total ms)} since profiling was enabled."""
    buf = (capi.BfmoeKernelTime * 64)()
    n = ctypes.c_int(0)
    capi.check(capi.lib().bfmoe_profile_collect(buf, 64, ctypes.byref(n)))
    return {buf[i].name.decode(): (buf[i].launches, buf[i].total_ms) for i in range(n.value)}


class ButterflyMoE:
    """Router + expert forward of one layer, with its own buffers.

    ``__call__(x)`` runs on device tensors; ``forward_host(x_host, y_host)``
    is the end-to-end call: pinned host tokens in, pinned host outputs back.
    """

    def __init__(self, layer: Layer, w_gate, bias, k: int, max_tokens: int, x_dtype):
        torch = _torch()
        self.layer, self.w_gate, self.bias, self.k = layer, w_gate, bias, k
        self.dtype = x_dtype
        code = BFMOE_BF16 if x_dtype == torch.bfloat16 else BFMOE_F32
        dev = layer.theta.device
        N, d = layer.n_experts, layer.d
        self.ws = workspace(d, N, max_tokens, k, code, dev)
        n = bfmoe_moe_workspace_size(d, N, max_tokens, k, code)
        self.ws_moe = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
        self.max_tokens = max_tokens
        self.idx = torch.empty((max_tokens, k), dtype=torch.int32, device=dev)
        self.gates = torch.empty((max_tokens, k), dtype=torch.float32, device=dev)
        self.counts = torch.empty((N,), dtype=torch.int32, device=dev)
        self.offsets = torch.empty((N + 1,), dtype=torch.int32, device=dev)
        self.rows = torch.empty((max_tokens * k,), dtype=torch.int32, device=dev)
        self.y_dev = torch.empty((max_tokens, d), dtype=x_dtype, device=dev)

    def route(self, x, stream=None):
        T = x.shape[0]
        out = (self.idx[:T], self.gates[:T], self.counts, self.offsets, self.rows[:T * self.k])
        return bfmoe_router_topk(x, self.w_gate, self.bias, self.k, self.ws, out=out, stream=stream)

    def __call__(self, x, y=None, stream=None):
        """Router + forward of x (device) through bfmoe_moe_forward."""
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError("more tokens than the buffers hold")
        if y is None:
            y = self.y_dev[:T]
        routing = (self.idx[:T], self.gates[:T], self.counts, self.offsets, self.rows[:T * self.k])
        y, _ = bfmoe_moe_forward(self.layer, x, self.w_gate, self.bias, self.k, self.ws_moe, routing=routing, y=y,
                                 stream=stream)
        return y

    def decode(self, x, y=None, stream=None):
        """Router (no buckets) + the add-only small-batch forward
        (bfmoe_decode_forward)."""
        T = x.shape[0]
        if T > self.max_tokens:
            raise ValueError("more tokens than the buffers hold")
        if y is None:
            y = self.y_dev[:T]
        idx, gates = self.idx[:T], self.gates[:T]
        bfmoe_router_topk(x, self.w_gate, self.bias, self.k, self.ws, out=(idx, gates, None, None, None),
                          stream=stream)
        return bfmoe_decode_forward(self.layer, x, self.k, idx, gates, y=y, stream=stream)

    def forward_host(self, x_host, y_host, chunk: int = 0, stream=None):
        """The end-to-end call: pinned host tokens in, pinned host outputs back,
        through bfmoe_moe_forward_host (copies overlapped with the work in
        token chunks).  Synchronise ``stream`` before reading y_host."""
        torch = _torch()
        T = x_host.shape[0]
        key = (T, chunk)
        if getattr(self, "_host_key", None) != key:
            code = BFMOE_BF16 if self.dtype == torch.bfloat16 else BFMOE_F32
            n = bfmoe_moe_host_workspace_size(self.layer.d, self.layer.n_experts, T, self.k, code, chunk)
            self.ws_host = torch.empty(max(n, 256), dtype=torch.uint8, device=self.layer.theta.device)
            self._host_key = key
        return bfmoe_moe_forward_host(self.layer, x_host, self.w_gate, self.bias, self.k, y_host, self.ws_host,
                                      chunk=chunk, stream=stream)
