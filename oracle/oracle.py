"""ctypes binding of the plain-C oracle (``moe_oracle.c``), numpy in and out.

TEST INFRASTRUCTURE ONLY (see the package docstring). Every function here is
a thin marshalling wrapper; the arithmetic is in ``moe_oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from .build import build as _build

_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = C.CDLL(_build())
        _declare(_lib)
    return _lib


def _p(a):
    return a.ctypes.data_as(C.c_void_p) if a is not None else None


def _declare(L):
    vp, i32, i64, dbl = C.c_void_p, C.c_int, C.c_int64, C.c_double
    L.oracle_bf16_to_double.argtypes = [C.c_uint16]
    L.oracle_bf16_to_double.restype = dbl
    L.oracle_bf16_from_double.argtypes = [dbl]
    L.oracle_bf16_from_double.restype = C.c_uint16
    L.oracle_e2m1_value.argtypes = [C.c_uint]
    L.oracle_e2m1_value.restype = dbl
    L.oracle_e8m0_value.argtypes = [C.c_uint]
    L.oracle_e8m0_value.restype = dbl
    L.oracle_e4m3_value.argtypes = [C.c_uint]
    L.oracle_e4m3_value.restype = dbl
    L.oracle_dequant_nvfp4.argtypes = [vp, vp, dbl, i64, vp]
    L.oracle_expert_nvfp4.argtypes = [vp, vp, vp, vp, i32, i32, vp, vp]
    L.oracle_moe_forward_nvfp4.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp,
                                           vp, vp, vp, vp, vp, vp]
    L.oracle_f16_value.argtypes = [C.c_uint]
    L.oracle_f16_value.restype = dbl
    L.oracle_dequant_sym8.argtypes = [vp, vp, i64, vp]
    L.oracle_expert_sym8.argtypes = [vp, vp, vp, i32, i32, vp, vp]
    L.oracle_moe_forward_sym8.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp,
                                          vp, vp, vp, vp, vp]
    L.oracle_dequant.argtypes = [vp, vp, i64, vp]
    L.oracle_dequant_f32.argtypes = [vp, vp, i64, vp]
    L.oracle_select_topk.argtypes = [vp, i32, i32, vp, vp]
    L.oracle_route.argtypes = [vp, i32, i32, vp, i32, vp, i32, vp, vp, vp]
    L.oracle_select_topk_sigmoid.argtypes = [vp, vp, i32, i32, vp, vp]
    L.oracle_route_sigmoid.argtypes = [vp, i32, i32, vp, i32, vp, i32, vp, vp, vp]
    L.oracle_expert.argtypes = [vp, vp, vp, i32, i32, vp, vp]
    L.oracle_combine.argtypes = [vp, vp, i32, i32, vp, vp]
    L.oracle_moe_forward.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp,
                                     vp, vp, vp, vp, vp]
    L.oracle_moe_layer.argtypes = [vp, i32, i32, i32, i32, i32, vp, vp, vp, vp,
                                   vp, vp, vp, vp]
    L.oracle_rmsnorm.argtypes = [vp, i32, i32, dbl, vp]
    L.oracle_stack_step.argtypes = [vp, i32, i32, i32, i32, i32, i32, vp, vp,
                                    vp, vp, dbl, vp]
    for name in ("oracle_dequant", "oracle_dequant_f32", "oracle_select_topk",
                 "oracle_select_topk_sigmoid", "oracle_route", "oracle_route_sigmoid",
                 "oracle_expert", "oracle_combine", "oracle_moe_forward", "oracle_moe_layer",
                 "oracle_dequant_nvfp4", "oracle_expert_nvfp4", "oracle_moe_forward_nvfp4",
                 "oracle_dequant_sym8", "oracle_expert_sym8", "oracle_moe_forward_sym8",
                 "oracle_rmsnorm",
                 "oracle_stack_step"):
        getattr(L, name).restype = None


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _gomp():
    lib()
    g = C.CDLL("libgomp.so.1")
    g.omp_get_max_threads.restype = C.c_int
    return g


def set_threads(n: int) -> None:
    """OpenMP thread count for the oracle's parallel loops."""
    _gomp().omp_set_num_threads(C.c_int(int(n)))


def max_threads() -> int:
    return int(_gomp().omp_get_max_threads())


# ------------------------------------------------------------------ scalars

def bf16_to_f64(b) -> float:
    return lib().oracle_bf16_to_double(int(b))


def bf16_from_f64(v) -> int:
    return int(lib().oracle_bf16_from_double(float(v)))


def e2m1_value(code: int) -> float:
    return lib().oracle_e2m1_value(int(code))


def e8m0_value(e: int) -> float:
    return lib().oracle_e8m0_value(int(e))


def e4m3_value(b: int) -> float:
    """FP8 E4M3 byte -> value (NVFP4 block scales)."""
    return lib().oracle_e4m3_value(int(b))


def f16_value(b: int) -> float:
    """IEEE binary16 bit pattern -> value (sym8 block scales)."""
    return lib().oracle_f16_value(int(b))


def bf16_from_f64_array(v: np.ndarray) -> np.ndarray:
    f = lib().oracle_bf16_from_double
    flat = np.asarray(v, dtype=np.float64).ravel()
    return np.array([f(float(a)) for a in flat], dtype=np.uint16).reshape(np.shape(v))


def bf16_to_f64_array(b: np.ndarray) -> np.ndarray:
    b = _c(b, np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


# ------------------------------------------------------------------ dequant

def dequant(codes: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    assert n % 32 == 0 and codes.size >= n // 2 and scales.size >= n // 32
    out = np.empty(n, dtype=np.float64)
    lib().oracle_dequant(_p(codes), _p(scales), n, _p(out))
    return out


def dequant_f32(codes: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    assert n % 32 == 0 and codes.size >= n // 2 and scales.size >= n // 32
    out = np.empty(n, dtype=np.float32)
    lib().oracle_dequant_f32(_p(codes), _p(scales), n, _p(out))
    return out


def dequant_nvfp4(codes: np.ndarray, scales: np.ndarray, gscale: float, n: int) -> np.ndarray:
    """NVFP4: E2M1 codes x E4M3 scale per 16 x global multiplier."""
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    assert n % 16 == 0 and codes.size >= n // 2 and scales.size >= n // 16
    out = np.empty(n, dtype=np.float64)
    lib().oracle_dequant_nvfp4(_p(codes), _p(scales), float(gscale), n, _p(out))
    return out


def dequant_sym8(q: np.ndarray, scales: np.ndarray, n: int) -> np.ndarray:
    """sym8: int8 q x binary16 scale per 32 (scales as uint16 words)."""
    q = _c(np.asarray(q).view(np.uint8), np.uint8)
    scales = _c(scales, np.uint16)
    assert n % 32 == 0 and q.size >= n and scales.size >= n // 32
    out = np.empty(n, dtype=np.float64)
    lib().oracle_dequant_sym8(_p(q), _p(scales), n, _p(out))
    return out


# ------------------------------------------------------------------- router

def select_topk(logits: np.ndarray, k: int):
    """Top-k + softmax of each row of logits [T, E] -> (ids [T,k], w [T,k])."""
    logits = _c(np.atleast_2d(logits), np.float64)
    T, E = logits.shape
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        lib().oracle_select_topk(_p(logits[t]), E, k, _p(ids[t]), _p(w[t]))
    return ids, w


def select_topk_sigmoid(logits: np.ndarray, bias, k: int):
    """Sigmoid scoring of each row of unbiased logits [T, E]: top-k of
    sigmoid(l) + bias, coefficients = the selected sigmoid scores over their
    sum -> (ids [T,k], w [T,k])."""
    logits = _c(np.atleast_2d(logits), np.float64)
    T, E = logits.shape
    b = _c(bias, np.float32) if bias is not None else None
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    for t in range(T):
        lib().oracle_select_topk_sigmoid(_p(logits[t]), _p(b), E, k, _p(ids[t]), _p(w[t]))
    return ids, w


def route(x, router_w, bias, k, sigmoid=False):
    """x bf16 [T,H], router_w bf16 [E,H], bias f32 [E] or None ->
    (ids int32 [T,k], w f64 [T,k], logits f64 [T,E]).  sigmoid: sigmoid
    scoring (logits unbiased, bias in the selection key only)."""
    x, router_w = _c(x, np.uint16), _c(router_w, np.uint16)
    T, H = x.shape
    E = router_w.shape[0]
    b = _c(bias, np.float32) if bias is not None else None
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    lg = np.empty((T, E), dtype=np.float64)
    fn = lib().oracle_route_sigmoid if sigmoid else lib().oracle_route
    fn(_p(x), T, H, _p(router_w), E, _p(b), k, _p(ids), _p(w), _p(lg))
    return ids, w, lg


# ------------------------------------------------------------------ experts

def expert(x, codes_e, scales_e, H, I):
    """One expert on one token -> (h bf16 [I], o bf16 [H])."""
    x = _c(x, np.uint16).ravel()
    codes_e, scales_e = _c(codes_e, np.uint8), _c(scales_e, np.uint8)
    h = np.empty(I, dtype=np.uint16)
    o = np.empty(H, dtype=np.uint16)
    lib().oracle_expert(_p(x), _p(codes_e), _p(scales_e), H, I, _p(h), _p(o))
    return h, o


def expert_nvfp4(x, codes_e, scales_e, gs, H, I):
    """One NVFP4 expert on one token -> (h bf16 [I], o bf16 [H]); gs =
    (gate/up multiplier, down multiplier)."""
    x = _c(x, np.uint16).ravel()
    codes_e, scales_e = _c(codes_e, np.uint8), _c(scales_e, np.uint8)
    gs = _c(gs, np.float32).ravel()
    h = np.empty(I, dtype=np.uint16)
    o = np.empty(H, dtype=np.uint16)
    lib().oracle_expert_nvfp4(_p(x), _p(codes_e), _p(scales_e), _p(gs), H, I, _p(h), _p(o))
    return h, o


def expert_sym8(x, q_e, scales_e, H, I):
    """One sym8 expert on one token -> (h bf16 [I], o bf16 [H]); q_e int8
    [3*I*H], scales_e binary16 words [3*I*H/32]."""
    x = _c(x, np.uint16).ravel()
    q_e = _c(np.asarray(q_e).view(np.uint8), np.uint8)
    scales_e = _c(scales_e, np.uint16)
    h = np.empty(I, dtype=np.uint16)
    o = np.empty(H, dtype=np.uint16)
    lib().oracle_expert_sym8(_p(x), _p(q_e), _p(scales_e), H, I, _p(h), _p(o))
    return h, o


def combine(o, w, residual=None):
    """o bf16 [k,H], w [k] -> y bf16 [H] (sequential BF16 combine)."""
    o = _c(o, np.uint16)
    k, H = o.shape
    w = _c(w, np.float64).ravel()
    r = _c(residual, np.uint16) if residual is not None else None
    y = np.empty(H, dtype=np.uint16)
    lib().oracle_combine(_p(o), _p(w), k, H, _p(r), _p(y))
    return y


def moe_forward_nvfp4(x, ids, w, codes, scales, gscales, E, H, I, residual=None,
                      want_o=False, want_h=False):
    """moe_forward for NVFP4 experts: scales [E, 3*I*H/16] E4M3 bytes,
    gscales [E, 2] float32 (gate/up, down)."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    w = _c(w, np.float64)
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    gscales = _c(gscales, np.float32)
    r = _c(residual, np.uint16) if residual is not None else None
    y = np.empty((T, H), dtype=np.uint16)
    o = np.empty((T, k, H), dtype=np.uint16) if want_o else None
    h = np.empty((T, k, I), dtype=np.uint16) if want_h else None
    lib().oracle_moe_forward_nvfp4(_p(x), T, E, H, I, k, _p(ids), _p(w), _p(codes),
                                   _p(scales), _p(gscales), _p(r), _p(y), _p(o), _p(h))
    out = [y]
    if want_o:
        out.append(o)
    if want_h:
        out.append(h)
    return out[0] if len(out) == 1 else tuple(out)


def moe_forward_sym8(x, ids, w, q, scales, E, H, I, residual=None,
                     want_o=False, want_h=False):
    """moe_forward for sym8 experts: q [E, 3*I*H] int8, scales [E, 3*I*H/32]
    binary16 words."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    w = _c(w, np.float64)
    q = _c(np.asarray(q).view(np.uint8), np.uint8)
    scales = _c(scales, np.uint16)
    r = _c(residual, np.uint16) if residual is not None else None
    y = np.empty((T, H), dtype=np.uint16)
    o = np.empty((T, k, H), dtype=np.uint16) if want_o else None
    h = np.empty((T, k, I), dtype=np.uint16) if want_h else None
    lib().oracle_moe_forward_sym8(_p(x), T, E, H, I, k, _p(ids), _p(w), _p(q), _p(scales),
                                  _p(r), _p(y), _p(o), _p(h))
    out = [y]
    if want_o:
        out.append(o)
    if want_h:
        out.append(h)
    return out[0] if len(out) == 1 else tuple(out)


def moe_forward(x, ids, w, codes, scales, E, H, I, residual=None,
                want_o=False, want_h=False):
    """Experts + combine for given routing. x bf16 [T,H], ids [T,k], w [T,k],
    codes [E, 3*I*H/2], scales [E, 3*I*H/32] -> y (and o [T,k,H], h [T,k,I])."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    ids = _c(ids, np.int32)
    k = ids.shape[1]
    w = _c(w, np.float64)
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    r = _c(residual, np.uint16) if residual is not None else None
    y = np.empty((T, H), dtype=np.uint16)
    o = np.empty((T, k, H), dtype=np.uint16) if want_o else None
    h = np.empty((T, k, I), dtype=np.uint16) if want_h else None
    lib().oracle_moe_forward(_p(x), T, E, H, I, k, _p(ids), _p(w), _p(codes),
                             _p(scales), _p(r), _p(y), _p(o), _p(h))
    out = [y]
    if want_o:
        out.append(o)
    if want_h:
        out.append(h)
    return out[0] if len(out) == 1 else tuple(out)


def moe_layer(x, router_w, bias, codes, scales, E, H, I, k, residual=None):
    """Route + experts + combine -> (ids, w, y)."""
    x = _c(x, np.uint16)
    T = x.shape[0]
    router_w = _c(router_w, np.uint16)
    b = _c(bias, np.float32) if bias is not None else None
    codes, scales = _c(codes, np.uint8), _c(scales, np.uint8)
    r = _c(residual, np.uint16) if residual is not None else None
    ids = np.empty((T, k), dtype=np.int32)
    w = np.empty((T, k), dtype=np.float64)
    y = np.empty((T, H), dtype=np.uint16)
    lib().oracle_moe_layer(_p(x), T, E, H, I, k, _p(router_w), _p(b), _p(codes),
                           _p(scales), _p(r), _p(ids), _p(w), _p(y))
    return ids, w, y


def rmsnorm(r, eps=1e-6):
    r = _c(np.atleast_2d(r), np.uint16)
    T, H = r.shape
    xn = np.empty_like(r)
    lib().oracle_rmsnorm(_p(r), T, H, float(eps), _p(xn))
    return xn


def stack_step(r, layers, eps=1e-6):
    """One decode step through the layers (list of workloads.LayerInputs).
    Returns (r_out bf16 [T,H], ids [L,T,k])."""
    r = _c(np.atleast_2d(r), np.uint16).copy()
    T, H = r.shape
    L = len(layers)
    sh = layers[0].shape
    keep = []
    Wr = (C.c_void_p * L)()
    Bs = (C.c_void_p * L)()
    Cs = (C.c_void_p * L)()
    Ss = (C.c_void_p * L)()
    any_bias = any(l.router_b is not None for l in layers)
    for i, l in enumerate(layers):
        a, c, s = _c(l.router_w, np.uint16), _c(l.codes, np.uint8), _c(l.scales, np.uint8)
        keep += [a, c, s]
        Wr[i], Cs[i], Ss[i] = a.ctypes.data, c.ctypes.data, s.ctypes.data
        if any_bias:
            b = _c(l.router_b, np.float32)
            keep.append(b)
            Bs[i] = b.ctypes.data
    ids = np.empty((L, T, sh.top_k), dtype=np.int32)
    lib().oracle_stack_step(_p(r), T, L, sh.E, H, sh.I, sh.top_k, Wr,
                            Bs if any_bias else None, Cs, Ss, float(eps), _p(ids))
    return r, ids
