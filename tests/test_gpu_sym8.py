"""sym8 experts (one int8 weight per element, one binary16 scale per 32 K
elements; page "LFM2.5-8B-A1B — Core AI (.aimodel)", table "Provenance", row
"Weight format") against the oracle: on the per-(token, slot) GEMV path
(up to 4 tokens, or in chunks when asked) the SwiGLU vectors h, expert
outputs o and combined y at the tolerance of the MXFP4 decode path; on the
grouped mma.sync products (beyond 4 tokens) at the grouped path's tolerance;
the combine bit-exact given the kernel's own o; invalid ids; the whole layer
(route, then the forward); argument errors."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import (assert_close_rms, check_grouped_y, dev_bf16, expert_matrix, host_bf16,
                      o_given_h, verify_h_flips)
from workloads import synth

pytestmark = pytest.mark.gpu


def _dev_sym8(L):
    q = torch.from_numpy(np.ascontiguousarray(L.codes)).cuda()
    s = torch.from_numpy(np.ascontiguousarray(L.scales).view(np.int16)).cuda()
    return q, s


def _layer(shape, seed, max_tokens=4, bias=False):
    L = synth.make_layer_sym8(shape, seed=seed, bias=bias)
    q, s = _dev_sym8(L)
    rb = None if L.router_b is None else torch.from_numpy(L.router_b).cuda()
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, q, s, dev_bf16(L.router_w), rb,
                         max_tokens=max_tokens)
    return L, layer


def _check(L, layer, x, ids, w, shape, residual=None):
    T = x.shape[0]
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=moe.FWD_KEEP_INTERMEDIATES,
                      residual=None if residual is None else dev_bf16(residual))
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    w64 = w.astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward_sym8(x, ids, w64, L.codes, L.scales, shape.E, shape.H,
                                            shape.I, residual=residual, want_o=True, want_h=True)
    valid = (ids >= 0) & (ids < shape.E)
    assert_close_rms(h_g[valid], h_r[valid], what="sym8 h")
    assert_close_rms(o_g[valid], o_r[valid], what="sym8 o")
    assert_close_rms(y_g, y_r, what="sym8 y", max_ulps=2)
    assert not o_g[~valid].any() and not h_g[~valid].any()
    for t in range(T):
        o_t = np.where(valid[t][:, None], o_g[t], 0).astype(np.uint16)
        want = oracle.combine(o_t, w64[t], None if residual is None else residual[t])
        np.testing.assert_array_equal(y_g[t], want)
    return y_g


@pytest.mark.parametrize("shape,T", [(synth.TINY, 1), (synth.TINY, 4), (synth.L24B, 1),
                                     (synth.L24B, 3), (synth.L8B, 1), (synth.L8B, 4)])
def test_sym8_forward_matches_oracle(shape, T):
    L, layer = _layer(shape, 71)
    x = synth.make_tokens(T, shape.H, seed=71, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(71, 13, T))
    r = synth.make_tokens(T, shape.H, seed=72, stream=T) if T > 1 else None
    _check(L, layer, x, ids, w, shape, residual=r)
    assert layer.status() == 0
    layer.close()


def _check_grouped(L, layer, x, ids, w, shape, flags=0, residual=None):
    """The grouped products stage by stage against the oracle (the
    tensor-core tiles sum the exact products in another FP32 order): every h
    element beyond 1e-2 rms a one-ulp rounding move of g, u or silu(g) at a
    midpoint; o against the oracle's down product of the kernel's own h; y by
    the bound the combine's arithmetic gives, and the combine bit-exact given
    the kernel's own o."""
    T = x.shape[0]
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=flags | moe.FWD_KEEP_INTERMEDIATES,
                      residual=None if residual is None else dev_bf16(residual))
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    w64 = w.astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward_sym8(x, ids, w64, L.codes, L.scales, shape.E, shape.H,
                                            shape.I, residual=residual, want_o=True, want_h=True)
    valid = (ids >= 0) & (ids < shape.E)
    matrix = lambda e, m: expert_matrix(L, shape, e, m, fmt="sym8")  # noqa: E731
    verify_h_flips(h_g, h_r, x, ids, valid, matrix, what="sym8 grouped h")
    o_ref = o_given_h(h_g, ids, valid, matrix, shape.H)
    assert_close_rms(o_g[valid], o_ref[valid], what="sym8 grouped o (given h)", max_ulps=2)
    check_grouped_y(y_g, y_r, o_g, o_r, w64, valid, residual, what="sym8 grouped y")
    for t in range(T):
        o_t = np.where(valid[t][:, None], o_g[t], 0).astype(np.uint16)
        want = oracle.combine(o_t, w64[t], None if residual is None else residual[t])
        np.testing.assert_array_equal(y_g[t], want)
    return y_g


@pytest.mark.parametrize("shape,T,dist", [
    (synth.TINY, 5, "uniform"), (synth.TINY, 33, "zipf"), (synth.TINY, 60, "uniform"),
    (synth.L24B, 5, "uniform"), (synth.L24B, 64, "uniform"), (synth.L24B, 64, "zipf"),
    (synth.L24B, 200, "uniform"), (synth.L8B, 17, "zipf")])
def test_sym8_grouped_matches_oracle(shape, T, dist):
    """Beyond the decode sizes sym8 experts run the (token, expert)-sorted
    grouped products (int8 rows converted to FP16 exactly on the tensor
    cores, the binary16 block scale applied per 32-element group in FP32):
    h, o and y against the oracle."""
    L, layer = _layer(shape, 79, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=79, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, dist, synth.rng_for(79, 13, T))
    r = synth.make_tokens(T, shape.H, seed=80, stream=T) if T % 2 else None
    _check_grouped(L, layer, x, ids, w, shape, residual=r)
    assert layer.status() == 0
    layer.close()


def test_sym8_grouped_and_per_pair_paths_both_hold():
    """The same batch on the grouped products (default beyond 4 tokens,
    FWD_FORCE_MMA, and FWD_FORCE_GROUPED at 3 tokens) and on the per-(token,
    slot) GEMVs in chunks (FWD_FORCE_DECODE), each against the oracle;
    invalid ids on the grouped path zero the slot and flag; the tcgen05
    products are refused; scales that are only 2-byte aligned keep the batch
    on the per-pair GEMVs (the grouped products are refused)."""
    shape = synth.TINY
    T = 11
    L, layer = _layer(shape, 73, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=73)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "zipf", synth.rng_for(73, 13, T))
    y_g = _check_grouped(L, layer, x, ids, w, shape)
    np.testing.assert_array_equal(_check_grouped(L, layer, x, ids, w, shape,
                                                 flags=moe.FWD_FORCE_MMA), y_g)
    y_d = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                        flags=moe.FWD_FORCE_DECODE | moe.FWD_KEEP_INTERMEDIATES)
    torch.cuda.synchronize()
    y_r = oracle.moe_forward_sym8(x, ids, w.astype(np.float64), L.codes, L.scales, shape.E,
                                  shape.H, shape.I)
    assert_close_rms(host_bf16(y_d), y_r, what="sym8 per-pair y", max_ulps=2)
    _check_grouped(L, layer, x[:3], ids[:3], w[:3], shape, flags=moe.FWD_FORCE_GROUPED)
    with pytest.raises(moe.MoEError):
        layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=moe.FWD_FORCE_TCGEN05)
    bad = ids.copy()
    bad[2, 1] = 99
    bad[7, 0] = -3
    _check_grouped(L, layer, x, bad, w, shape)
    assert layer.status() & moe.DEVICE_BAD_EXPERT_ID
    layer.close()

    q, s = _dev_sym8(L)
    pool = torch.zeros(s.numel() + 8, dtype=torch.int16, device="cuda")
    s2 = pool[1:1 + s.numel()].view(s.shape)  # 2-byte aligned only
    s2.copy_(s)
    rw = dev_bf16(L.router_w)
    layer2 = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, q, s2, rw, None, max_tokens=T)
    _check(L, layer2, x, ids, w, shape)
    with pytest.raises(moe.MoEError):
        layer2.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                       flags=moe.FWD_FORCE_GROUPED)
    layer2.close()


def test_sym8_invalid_ids_zero_the_slot_and_flag():
    shape = synth.TINY
    L, layer = _layer(shape, 74)
    x = synth.make_tokens(3, shape.H, seed=74)
    ids, w = synth.make_routing(3, shape.E, shape.top_k, "uniform", synth.rng_for(74, 13, 3))
    ids[1, 2] = 77
    ids[2, 0] = -5
    _check(L, layer, x, ids, w, shape)
    assert layer.status() & moe.DEVICE_BAD_EXPERT_ID
    layer.close()


def test_sym8_deterministic_and_phase_split():
    """Two runs give the same bits; the gate/up and down launches run apart
    (phase flags) give the bits of the whole forward."""
    shape = synth.L24B
    L, layer = _layer(shape, 75)
    T = 2
    x = dev_bf16(synth.make_tokens(T, shape.H, seed=75))
    ids_h, w_h = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(75, 13, T))
    ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
    y1 = host_bf16(layer.forward(x, ids, w)).copy()
    y2 = host_bf16(layer.forward(x, ids, w)).copy()
    y3 = torch.zeros_like(x)
    layer.forward(x, ids, w, y=y3, flags=moe.FWD_PHASE_GATEUP)
    layer.forward(x, ids, w, y=y3, flags=moe.FWD_PHASE_DOWN)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y1, y2)
    np.testing.assert_array_equal(y1, host_bf16(y3))
    layer.close()


def test_sym8_layer_is_route_then_forward():
    """moe_layer_ex on sym8 experts (every fusion setting runs the separate
    launches) gives the bits of moe_route_ex + moe_forward_ex, and the layer
    output matches the oracle fed the GPU's normalised input and routing."""
    shape = synth.L8B
    L, layer = _layer(shape, 76, bias=True)
    T = 2
    xr = dev_bf16(synth.make_tokens(T, shape.H, seed=76))
    res = dev_bf16(synth.make_tokens(T, shape.H, seed=77))
    outs = []
    for mode in ("layer", moe.FUSION_NONE, moe.FUSION_ROUTER, moe.FUSION_LAYER):
        xn = torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda")
        ids = torch.zeros(T, shape.top_k, dtype=torch.int32, device="cuda")
        w = torch.zeros(T, shape.top_k, dtype=torch.float32, device="cuda")
        y = torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda")
        if mode == "layer":
            moe.moe_route_ex(layer.handle, xr, layer.router_w, layer.router_b,
                             moe.ROUTE_RMSNORM, xn, None, ids, w)
            moe.moe_forward_ex(layer.handle, xn, ids, w, res, y, 0)
        else:
            moe.moe_set_fusion(layer.handle, mode)
            moe.moe_layer_ex(layer.handle, xr, layer.router_w, layer.router_b,
                             moe.ROUTE_RMSNORM, xn, None, ids, w, res, y, 0)
        torch.cuda.synchronize()
        assert layer.status() == 0
        outs.append([host_bf16(xn).copy(), ids.cpu().numpy(), w.cpu().numpy(),
                     host_bf16(y).copy()])
    for o in outs[1:]:
        for a, b in zip(outs[0], o):
            np.testing.assert_array_equal(a, b)
    xn_h, ids_h, w_h, y_h = outs[0]
    y_r = oracle.moe_forward_sym8(xn_h, ids_h, w_h.astype(np.float64), L.codes, L.scales,
                                  shape.E, shape.H, shape.I, residual=host_bf16(res))
    assert_close_rms(y_h, y_r, what="sym8 layer y", max_ulps=2)
    layer.close()


def test_sym8_argument_errors():
    """Shapes outside the kernels' set, a misaligned code pointer, and the
    one-launch stack (MXFP4 and NVFP4 layers only) are refused."""
    # top_k * I BF16 values of h (8 * 4096 * 2 bytes) beyond the staged 48 KB
    bad = synth.LayerShape(E=8, H=512, I=4096, top_k=8)
    h = moe.moe_create(bad.E, bad.H, bad.I, bad.top_k)
    try:
        q = torch.zeros(bad.E * 3 * bad.I * bad.H, dtype=torch.int8, device="cuda")
        s = torch.zeros(bad.E * 3 * bad.I * bad.H // 32, dtype=torch.int16, device="cuda")
        with pytest.raises(moe.MoEError):
            moe.moe_load_packed_sym8(h, q, s)
    finally:
        moe.moe_destroy(h)
    shape = synth.TINY
    L = synth.make_layer_sym8(shape, seed=78)
    q, s = _dev_sym8(L)
    h = moe.moe_create(shape.E, shape.H, shape.I, shape.top_k)
    try:
        pool = torch.zeros(q.numel() + 16, dtype=torch.int8, device="cuda")
        with pytest.raises(moe.MoEError):
            moe.moe_load_packed_sym8(h, pool[1:1 + q.numel()], s)
    finally:
        moe.moe_destroy(h)
    _, layer = _layer(shape, 78)
    with pytest.raises(moe.MoEError):
        moe.MoEStack([(q, s, dev_bf16(L.router_w), None)], shape.E, shape.H, shape.I,
                     shape.top_k, persistent=True)
    layer.close()
