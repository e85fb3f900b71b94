"""Packed-MXFP4 W4A16 top-4 MoE expert FFN for NVIDIA B200 (sm_100a).

Python binding of the C-ABI library ``libmoe_mxfp4.so`` (declared in
``include/moe_mxfp4.h``). The functions below carry the C names and only
marshal arguments: torch tensors give device pointers, the current torch
stream gives the CUDA stream, every step of the computation runs in the
library's kernels. There is no CPU fallback: if the library is missing or the
device is not sm_100, the calls raise.

``MoELayer`` and ``MoEStack`` bundle the calls with their buffers: a single
layer (route + experts + combine) and a stack of layers (weightless RMSNorm,
route, experts, combine with residual add, per layer) captured in one CUDA
graph per decode step.
"""
from __future__ import annotations

import ctypes as C

import torch

from ._lib import MoEError, check, library_path, load

__all__ = [
    "MoEError", "MoELayer", "MoEStack", "library_path", "load",
    "moe_create", "moe_destroy", "moe_load_packed", "moe_load_packed_nvfp4", "moe_load_packed_sym8",
    "moe_load_expert_table",
    "moe_workspace_bytes", "moe_set_workspace", "moe_route", "moe_route_ex",
    "moe_forward", "moe_forward_ex", "moe_layer_ex", "moe_get_intermediates", "moe_get_status", "moe_get_status_stream",
    "moe_bytes_per_expert", "moe_set_tuning", "moe_device_check", "moe_debug_dequant",
    "moe_forward_noalloc", "moe_forward_noalloc_status", "moe_stack_create", "moe_stack_destroy", "moe_stack_workspace_bytes",
    "moe_stack_set_workspace", "moe_stack_decode", "moe_stack_get_status",
    "moe_stack_set_spin_limit", "moe_stack_set_trace", "STACK_TRACE_SLOTS",
    "ROUTE_RMSNORM", "ROUTE_SIGMOID", "FWD_KEEP_INTERMEDIATES", "FWD_FORCE_DECODE", "FWD_FORCE_GROUPED",
    "FWD_PHASE_GATEUP", "FWD_PHASE_DOWN", "FWD_FORCE_TCGEN05", "FWD_FORCE_MMA",
    "FUSION_NONE", "FUSION_ROUTER", "FUSION_LAYER", "moe_set_fusion",
    "DEVICE_BAD_EXPERT_ID",
]

ROUTE_RMSNORM = 0x1
ROUTE_SIGMOID = 0x2
FWD_KEEP_INTERMEDIATES = 0x1
FWD_FORCE_DECODE = 0x2
FWD_FORCE_GROUPED = 0x4
FWD_PHASE_GATEUP = 0x8
FWD_PHASE_DOWN = 0x10
FWD_FORCE_TCGEN05 = 0x20
FWD_FORCE_MMA = 0x40
FUSION_NONE, FUSION_ROUTER, FUSION_LAYER = 0, 1, 2
DEVICE_BAD_EXPERT_ID = 0x1
DEVICE_TIMEOUT = 0x2


def _p(t):
    return None if t is None else C.c_void_p(t.data_ptr())


def _s(stream):
    s = stream if stream is not None else torch.cuda.current_stream()
    return C.c_void_p(s.cuda_stream)


def _need(t, dtype, name, ndim=None):
    if t is None:
        return
    if not t.is_cuda or t.dtype != dtype or not t.is_contiguous():
        raise MoEError(name, -1)
    if ndim is not None and t.dim() != ndim:
        raise MoEError(name, -1)


# ------------------------------------------------------------ C-ABI names

def moe_create(E: int, H: int, I: int, top_k: int) -> int:
    h = C.c_void_p()
    check("moe_create", load().moe_create(E, H, I, top_k, C.byref(h)))
    return h.value


def moe_destroy(h: int) -> None:
    check("moe_destroy", load().moe_destroy(C.c_void_p(h)))


def moe_load_packed(h: int, codes: torch.Tensor, scales: torch.Tensor) -> None:
    _need(codes, torch.uint8, "moe_load_packed")
    _need(scales, torch.uint8, "moe_load_packed")
    check("moe_load_packed", load().moe_load_packed(C.c_void_p(h), _p(codes), _p(scales)))


def moe_load_packed_nvfp4(h: int, codes: torch.Tensor, scales: torch.Tensor,
                          gscales: torch.Tensor) -> None:
    """NVFP4 experts: codes uint8 [E, 3*I*H/2], E4M3 scales uint8
    [E, 3*I*H/16], multipliers float32 [E, 2] (gate/up, down)."""
    _need(codes, torch.uint8, "moe_load_packed_nvfp4")
    _need(scales, torch.uint8, "moe_load_packed_nvfp4")
    _need(gscales, torch.float32, "moe_load_packed_nvfp4")
    check("moe_load_packed_nvfp4",
          load().moe_load_packed_nvfp4(C.c_void_p(h), _p(codes), _p(scales), _p(gscales)))


def moe_load_packed_sym8(h: int, codes: torch.Tensor, scales: torch.Tensor) -> None:
    """sym8 experts: codes int8 [E, 3*I*H] (one byte per weight), scales
    binary16 words [E, 3*I*H/32] (a float16 or int16/uint16 tensor of the bit
    patterns)."""
    _need(codes, torch.int8, "moe_load_packed_sym8")
    if (scales.dtype not in (torch.float16, torch.int16, torch.uint16) or not scales.is_cuda
            or not scales.is_contiguous()):
        raise MoEError("moe_load_packed_sym8", -1)
    check("moe_load_packed_sym8",
          load().moe_load_packed_sym8(C.c_void_p(h), _p(codes), _p(scales)))


def moe_load_expert_table(h: int, codes_ptrs, scales_ptrs) -> None:
    """codes_ptrs / scales_ptrs: sequences of 3*E device addresses (ints)."""
    n = len(codes_ptrs)
    ca = (C.c_void_p * n)(*codes_ptrs)
    sa = (C.c_void_p * n)(*scales_ptrs)
    check("moe_load_expert_table", load().moe_load_expert_table(C.c_void_p(h), ca, sa))


def moe_workspace_bytes(h: int, max_tokens: int) -> int:
    n = C.c_size_t()
    check("moe_workspace_bytes", load().moe_workspace_bytes(C.c_void_p(h), max_tokens, C.byref(n)))
    return n.value


def moe_set_workspace(h: int, ws: torch.Tensor, max_tokens: int) -> None:
    _need(ws, torch.uint8, "moe_set_workspace")
    check("moe_set_workspace",
          load().moe_set_workspace(C.c_void_p(h), _p(ws), ws.numel(), max_tokens))


def moe_route(h, x, router_w, router_bias, topk_ids, topk_w, stream=None) -> None:
    moe_route_ex(h, x, router_w, router_bias, 0, None, None, topk_ids, topk_w, stream)


def moe_route_ex(h, x, router_w, router_bias, flags, x_norm, logits, topk_ids, topk_w,
                 stream=None) -> None:
    _need(x, torch.bfloat16, "moe_route", 2)
    _need(router_w, torch.bfloat16, "moe_route", 2)
    _need(router_bias, torch.float32, "moe_route")
    _need(x_norm, torch.bfloat16, "moe_route")
    _need(logits, torch.float32, "moe_route")
    _need(topk_ids, torch.int32, "moe_route")
    _need(topk_w, torch.float32, "moe_route")
    check("moe_route", load().moe_route_ex(
        C.c_void_p(h), _p(x), x.shape[0], _p(router_w), _p(router_bias), flags, _p(x_norm),
        _p(logits), _p(topk_ids), _p(topk_w), _s(stream)))


def moe_forward(h, x, topk_ids, topk_w, y, stream=None) -> None:
    moe_forward_ex(h, x, topk_ids, topk_w, None, y, 0, stream)


def moe_forward_ex(h, x, topk_ids, topk_w, residual, y, flags, stream=None) -> None:
    _need(x, torch.bfloat16, "moe_forward", 2)
    _need(topk_ids, torch.int32, "moe_forward")
    _need(topk_w, torch.float32, "moe_forward")
    _need(residual, torch.bfloat16, "moe_forward")
    _need(y, torch.bfloat16, "moe_forward")
    check("moe_forward", load().moe_forward_ex(
        C.c_void_p(h), _p(x), x.shape[0], _p(topk_ids), _p(topk_w), _p(residual), _p(y),
        flags, _s(stream)))


def moe_layer_ex(h, x, router_w, router_bias, route_flags, x_norm, logits, topk_ids, topk_w,
                 residual, y, fwd_flags, stream=None) -> None:
    _need(x, torch.bfloat16, "moe_layer_ex", 2)
    _need(router_w, torch.bfloat16, "moe_layer_ex", 2)
    _need(router_bias, torch.float32, "moe_layer_ex")
    _need(x_norm, torch.bfloat16, "moe_layer_ex")
    _need(logits, torch.float32, "moe_layer_ex")
    _need(topk_ids, torch.int32, "moe_layer_ex")
    _need(topk_w, torch.float32, "moe_layer_ex")
    _need(residual, torch.bfloat16, "moe_layer_ex")
    _need(y, torch.bfloat16, "moe_layer_ex")
    check("moe_layer_ex", load().moe_layer_ex(
        C.c_void_p(h), _p(x), x.shape[0], _p(router_w), _p(router_bias), route_flags,
        _p(x_norm), _p(logits), _p(topk_ids), _p(topk_w), _p(residual), _p(y), fwd_flags,
        _s(stream)))


def moe_get_intermediates(h: int):
    """Device addresses (h_ptr, o_ptr) of the intermediates of the last forward
    run with FWD_KEEP_INTERMEDIATES."""
    hp, op = C.c_void_p(), C.c_void_p()
    check("moe_get_intermediates",
          load().moe_get_intermediates(C.c_void_p(h), C.byref(hp), C.byref(op)))
    return hp.value, op.value


def moe_get_status(h: int) -> int:
    v = C.c_uint()
    check("moe_get_status", load().moe_get_status(C.c_void_p(h), C.byref(v)))
    return v.value


def moe_get_status_stream(h: int, stream=None) -> int:
    """Device status of the handle's work on `stream` (torch stream or None:
    the current stream), cleared; waits for that stream only."""
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    v = C.c_uint()
    check("moe_get_status_stream",
          load().moe_get_status_stream(C.c_void_p(h), C.c_void_p(s.cuda_stream), C.byref(v)))
    return v.value


def moe_bytes_per_expert(h: int) -> int:
    n = C.c_size_t()
    check("moe_bytes_per_expert", load().moe_bytes_per_expert(C.c_void_p(h), C.byref(n)))
    return n.value


def moe_set_tuning(h: int, use_pdl: bool, prefetch_down: bool) -> None:
    check("moe_set_tuning", load().moe_set_tuning(C.c_void_p(h), int(use_pdl), int(prefetch_down)))


def moe_set_fusion(h: int, mode: int) -> None:
    check("moe_set_fusion", load().moe_set_fusion(C.c_void_p(h), int(mode)))


def moe_device_check() -> None:
    check("moe_device_check", load().moe_device_check())


def moe_debug_dequant(codes, scales, n, out, stream=None) -> None:
    _need(codes, torch.uint8, "moe_debug_dequant")
    _need(scales, torch.uint8, "moe_debug_dequant")
    _need(out, torch.float32, "moe_debug_dequant")
    check("moe_debug_dequant", load().moe_debug_dequant(_p(codes), _p(scales), n, _p(out), _s(stream)))


def _noalloc_args_ok(E, H, I, top_k, codes, scales, x, topk_ids, topk_w, residual, y,
                     device=None):
    """Shape, dtype, layout and device checks of moe_forward_noalloc's tensors
    (the C call takes bare pointers and cannot check sizes).  Raises MoEError
    (MOE_ERR_ARG) on a mismatch.  `device`: the device every tensor must be on
    (default: the current CUDA device)."""
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    device = torch.device(device)

    def need(t, dtype, numel, what):
        ok = (t is not None and t.dtype == dtype and t.is_contiguous() and t.numel() == numel
              and t.device == device)
        if not ok:
            raise MoEError(f"moe_forward_noalloc ({what})", -1)

    if x is None or x.dim() != 2 or x.shape[1] != H:
        raise MoEError("moe_forward_noalloc (x shape)", -1)
    T = x.shape[0]
    need(codes, torch.uint8, E * 3 * I * H // 2, "codes")
    need(scales, torch.uint8, E * 3 * I * H // 32, "scales")
    need(x, torch.bfloat16, T * H, "x")
    need(topk_ids, torch.int32, T * top_k, "topk_ids")
    need(topk_w, torch.float32, T * top_k, "topk_w")
    need(y, torch.bfloat16, T * H, "y")
    if residual is not None:
        need(residual, torch.bfloat16, T * H, "residual")
    return T


def moe_forward_noalloc(E, H, I, top_k, codes, scales, x, topk_ids, topk_w, residual, y,
                        stream=None) -> None:
    """Expert FFN + combine for callers that may not allocate device memory:
    no handle, no workspace; scratch lives in a fixed device array inside the
    library (see include/moe_mxfp4.h for its limits and its sharing rules).
    Every tensor is checked against E, H, I, top_k and T = x.shape[0] and must
    be on the current device."""
    T = _noalloc_args_ok(E, H, I, top_k, codes, scales, x, topk_ids, topk_w, residual, y)
    check("moe_forward_noalloc", load().moe_forward_noalloc(
        E, H, I, top_k, _p(codes), _p(scales), _p(x), T, _p(topk_ids), _p(topk_w),
        _p(residual), _p(y), _s(stream)))


def moe_forward_noalloc_status(stream=None) -> int:
    """Status bits of moe_forward_noalloc on the current device since the
    last read (synchronises `stream`), cleared."""
    v = C.c_uint()
    check("moe_forward_noalloc_status", load().moe_forward_noalloc_status(_s(stream), C.byref(v)))
    return v.value


def moe_stack_create(handles, router_ws, router_bs=None) -> int:
    """A decode stack over layer handles (ints); router_ws / router_bs:
    sequences of device tensors (BF16 [E, H]; FP32 [E] or None)."""
    n = len(handles)
    for t in router_ws:
        _need(t, torch.bfloat16, "moe_stack_create", 2)
    ha = (C.c_void_p * n)(*handles)
    wa = (C.c_void_p * n)(*[t.data_ptr() for t in router_ws])
    ba = None
    if router_bs is not None and any(b is not None for b in router_bs):
        for t in router_bs:
            _need(t, torch.float32, "moe_stack_create")
        ba = (C.c_void_p * n)(*[None if b is None else b.data_ptr() for b in router_bs])
    out = C.c_void_p()
    check("moe_stack_create", load().moe_stack_create(ha, n, wa, ba, C.byref(out)))
    return out.value


def moe_stack_destroy(s: int) -> None:
    check("moe_stack_destroy", load().moe_stack_destroy(C.c_void_p(s)))


def moe_stack_workspace_bytes(s: int) -> int:
    n = C.c_size_t()
    check("moe_stack_workspace_bytes", load().moe_stack_workspace_bytes(C.c_void_p(s), C.byref(n)))
    return n.value


def moe_stack_set_workspace(s: int, ws: torch.Tensor) -> None:
    _need(ws, torch.uint8, "moe_stack_set_workspace")
    check("moe_stack_set_workspace", load().moe_stack_set_workspace(C.c_void_p(s), _p(ws), ws.numel()))


def moe_stack_decode(s, r, r_hist=None, xn_hist=None, logits=None, topk_ids=None, topk_w=None,
                     stream=None) -> None:
    _need(r, torch.bfloat16, "moe_stack_decode")
    _need(r_hist, torch.bfloat16, "moe_stack_decode")
    _need(xn_hist, torch.bfloat16, "moe_stack_decode")
    _need(logits, torch.float32, "moe_stack_decode")
    _need(topk_ids, torch.int32, "moe_stack_decode")
    _need(topk_w, torch.float32, "moe_stack_decode")
    check("moe_stack_decode", load().moe_stack_decode(
        C.c_void_p(s), _p(r), _p(r_hist), _p(xn_hist), _p(logits), _p(topk_ids), _p(topk_w),
        _s(stream)))


def moe_stack_get_status(s: int, stream=None) -> int:
    v = C.c_uint()
    check("moe_stack_get_status", load().moe_stack_get_status(C.c_void_p(s), _s(stream), C.byref(v)))
    return v.value


STACK_TRACE_SLOTS = 16


def moe_stack_set_trace(s: int, trace) -> None:
    """trace: device int64 tensor of n_layers * SMs * STACK_TRACE_SLOTS
    elements (phase time stamps of every later decode), or None."""
    if trace is None:
        check("moe_stack_set_trace", load().moe_stack_set_trace(C.c_void_p(s), None, 0))
        return
    _need(trace, torch.int64, "moe_stack_set_trace")
    check("moe_stack_set_trace",
          load().moe_stack_set_trace(C.c_void_p(s), _p(trace), trace.numel() * 8))


def moe_stack_set_spin_limit(s: int, polls: int) -> None:
    check("moe_stack_set_spin_limit", load().moe_stack_set_spin_limit(C.c_void_p(s), int(polls)))


# ------------------------------------------------------------- bundles

class MoELayer:
    """One MoE layer bound to packed weights already on the device.

    codes uint8 [E, 3*I*H/2] and scales uint8 [E, 3*I*H/32] (layout of
    include/moe_mxfp4.h) are read in place; the layer keeps references to
    them. ``router_w`` BF16 [E, H], ``router_b`` FP32 [E] or None.  With
    ``gscales`` (float32 [E, 2]) the experts are NVFP4: scales are then E4M3
    bytes [E, 3*I*H/16].  With int8 ``codes`` [E, 3*I*H] the experts are
    sym8: scales are then binary16 words [E, 3*I*H/32].
    """

    def __init__(self, E, H, I, top_k, codes, scales, router_w=None, router_b=None,
                 max_tokens=4, workspace=None, gscales=None):
        moe_device_check()
        self.E, self.H, self.I, self.k = E, H, I, top_k
        self.codes, self.scales, self.gscales = codes, scales, gscales
        self.router_w, self.router_b = router_w, router_b
        self.max_tokens = max_tokens
        self.handle = moe_create(E, H, I, top_k)
        try:
            if codes.dtype == torch.int8:
                moe_load_packed_sym8(self.handle, codes, scales)
            elif gscales is None:
                moe_load_packed(self.handle, codes, scales)
            else:
                moe_load_packed_nvfp4(self.handle, codes, scales, gscales)
            need = moe_workspace_bytes(self.handle, max_tokens)
            if workspace is None:
                workspace = torch.empty(need, dtype=torch.uint8, device=codes.device)
            self.workspace = workspace
            moe_set_workspace(self.handle, workspace, max_tokens)
        except Exception:
            moe_destroy(self.handle)
            self.handle = None
            raise

    def close(self):
        if getattr(self, "handle", None):
            moe_destroy(self.handle)
            self.handle = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def route(self, x, ids=None, w=None, logits=None, x_norm=None, rmsnorm=False, sigmoid=False,
              stream=None):
        T = x.shape[0]
        dev = x.device
        ids = ids if ids is not None else torch.empty(T, self.k, dtype=torch.int32, device=dev)
        w = w if w is not None else torch.empty(T, self.k, dtype=torch.float32, device=dev)
        flags = (ROUTE_RMSNORM if rmsnorm else 0) | (ROUTE_SIGMOID if sigmoid else 0)
        if rmsnorm and x_norm is None:
            x_norm = torch.empty_like(x)
        moe_route_ex(self.handle, x, self.router_w, self.router_b, flags,
                     x_norm if rmsnorm else None, logits, ids, w, stream)
        return (ids, w, x_norm) if rmsnorm else (ids, w)

    def forward(self, x, ids, w, y=None, residual=None, flags=0, stream=None):
        y = y if y is not None else torch.empty_like(x)
        moe_forward_ex(self.handle, x, ids, w, residual, y, flags, stream)
        return y

    def __call__(self, x, stream=None):
        ids, w = self.route(x, stream=stream)
        return self.forward(x, ids, w, stream=stream)

    def intermediates(self, T):
        """Views (h [T,k,I], o [T,k,H], BF16) into the workspace of the last
        forward run with FWD_KEEP_INTERMEDIATES."""
        hp, op = moe_get_intermediates(self.handle)
        base = self.workspace.data_ptr()
        hv = self.workspace[hp - base: hp - base + T * self.k * self.I * 2]
        ov = self.workspace[op - base: op - base + T * self.k * self.H * 2]
        return (hv.view(torch.bfloat16).view(T, self.k, self.I),
                ov.view(torch.bfloat16).view(T, self.k, self.H))

    def status(self, stream=None) -> int:
        """Device status bits (cleared).  With a stream: waits for that stream
        only; without: for the whole device."""
        if stream is not None:
            return moe_get_status_stream(self.handle, stream)
        return moe_get_status(self.handle)


class MoEStack:
    """A stack of MoE layers run as one decode step on a residual stream r:
    per layer xn = RMSNorm(r) (weightless, eps 1e-6), route(xn), experts,
    r = BF16(r + combine).  ``step()`` replays one CUDA graph of all layers.
    Layers share one workspace (they run in order on one stream).
    ``layers_weights``: per layer (codes, scales, router_w, router_b), or
    with a fifth item, the NVFP4 multipliers [E, 2] (see MoELayer).

    ``persistent``: run the whole step as one launch (moe_stack_decode);
    None = when the shape allows it (T = 1, MXFP4 layers, shapes of
    moe_stack_create), False = one layer at a time (moe_layer_ex), True =
    required."""

    def __init__(self, layers_weights, E, H, I, top_k, T=1, device="cuda", persistent=None):
        moe_device_check()
        self.E, self.H, self.I, self.k, self.T = E, H, I, top_k, T
        self.layers = []
        ws = None
        for lw in layers_weights:
            codes, scales, router_w, router_b = lw[:4]
            gscales = lw[4] if len(lw) > 4 else None
            L = MoELayer(E, H, I, top_k, codes, scales, router_w, router_b, max_tokens=T,
                         workspace=ws, gscales=gscales)
            ws = L.workspace
            self.layers.append(L)
        dev = torch.device(device)
        n = len(self.layers)
        self.r = torch.zeros(T, H, dtype=torch.bfloat16, device=dev)
        self.xn = torch.zeros(T, H, dtype=torch.bfloat16, device=dev)
        self.ids = torch.zeros(n, T, top_k, dtype=torch.int32, device=dev)
        self.w = torch.zeros(n, T, top_k, dtype=torch.float32, device=dev)
        self.graph = None
        self.stream = torch.cuda.Stream(device=dev)
        # one launch for the whole step (moe_stack_*) when the shape allows it
        self.stack = None
        self.stack_ws = None
        if persistent is not False and T == 1:
            try:
                self.stack = moe_stack_create([L.handle for L in self.layers],
                                              [L.router_w for L in self.layers],
                                              [L.router_b for L in self.layers])
                self.stack_ws = torch.empty(moe_stack_workspace_bytes(self.stack),
                                            dtype=torch.uint8, device=dev)
                moe_stack_set_workspace(self.stack, self.stack_ws)
            except MoEError:
                if self.stack is not None:
                    moe_stack_destroy(self.stack)
                self.stack = None
                if persistent:
                    raise
        elif persistent:
            raise MoEError("moe_stack_create", -1)

    def set_tuning(self, use_pdl=True, prefetch_down=True):
        for L in self.layers:
            moe_set_tuning(L.handle, use_pdl, prefetch_down)

    def set_fusion(self, mode):
        """Launch structure of every layer (FUSION_NONE / _ROUTER / _LAYER)."""
        for L in self.layers:
            moe_set_fusion(L.handle, mode)

    def enqueue(self, stream=None):
        """Enqueue one decode step (all layers) on `stream`."""
        if self.stack is not None:
            moe_stack_decode(self.stack, self.r, topk_ids=self.ids, topk_w=self.w, stream=stream)
        else:
            self.enqueue_layers(stream)

    def enqueue_layers(self, stream=None):
        """The same step as one moe_layer_ex call per layer."""
        for l, L in enumerate(self.layers):
            moe_layer_ex(L.handle, self.r, L.router_w, L.router_b, ROUTE_RMSNORM, self.xn, None,
                         self.ids[l], self.w[l], self.r, self.r, 0, stream)

    def status(self, stream=None) -> int:
        """Device status bits of the stack kernel and of every layer handle
        (synchronises), cleared."""
        st = 0
        if self.stack is not None:
            st |= moe_stack_get_status(self.stack, stream)
        for L in self.layers:
            st |= L.status()
        return st

    def capture(self):
        """Capture one decode step into a CUDA graph (warm-up run first)."""
        s = self.stream
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):
            saved = self.r.clone()
            self.enqueue(s)
            self.r.copy_(saved)
        torch.cuda.current_stream().wait_stream(s)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            self.enqueue(s)
        self.graph = g
        return g

    def step(self):
        """One decode step: replay the captured graph (captures on first use)."""
        if self.graph is None:
            self.capture()
        self.graph.replay()

    def decode_host(self, x_host, y_host):
        """Decode the tokens of x_host one step each (T rows per step) from
        host memory: per step, copy its input into the residual stream,
        replay the captured step, copy the residual stream back into y_host.
        Returns after the last copy has landed.  Pinned buffers make the
        copies asynchronous."""
        if self.graph is None:
            self.capture()
        T = self.T
        for i in range(x_host.shape[0] // T):
            self.r.copy_(x_host[i * T:(i + 1) * T], non_blocking=True)
            self.graph.replay()
            y_host[i * T:(i + 1) * T].copy_(self.r, non_blocking=True)
        torch.cuda.current_stream().synchronize()
        return y_host

    def close(self):
        self.graph = None
        if getattr(self, "stack", None) is not None:
            moe_stack_destroy(self.stack)
            self.stack = None
        for L in self.layers:
            L.close()
