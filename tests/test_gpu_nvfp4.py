"""NVFP4 experts (E2M1 codes, an FP8 E4M3 scale per 16 elements, an FP32
multiplier per expert for gate/up and one for down) against the oracle: the
per-(token, slot) path (T <= 4), the grouped mma.sync products (larger T,
or forced) and the grouped tcgen05 products (large groups, or forced) —
SwiGLU vectors h, expert outputs o and combined y at the tolerance of the
MXFP4 paths; the combine bit-exact given the kernel's own o; uniform and
Zipf routing; invalid ids; the whole layer; argument errors."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import (assert_close_rms, check_grouped_y, dev_bf16, dev_u8, expert_matrix,
                      host_bf16, o_given_h, verify_h_flips)
from workloads import synth

pytestmark = pytest.mark.gpu


def _layer(shape, seed, max_tokens=4, bias=False):
    L = synth.make_layer_nvfp4(shape, seed=seed, bias=bias)
    rb = None if L.router_b is None else torch.from_numpy(L.router_b).cuda()
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, dev_u8(L.codes),
                         dev_u8(L.scales), dev_bf16(L.router_w), rb, max_tokens=max_tokens,
                         gscales=torch.from_numpy(L.gscales).cuda())
    return L, layer


def _check(L, layer, x, ids, w, shape, residual=None, flags=0, ulps=1, h_ulps=None):
    T = x.shape[0]
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=moe.FWD_KEEP_INTERMEDIATES | flags,
                      residual=None if residual is None else dev_bf16(residual))
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    w64 = w.astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward_nvfp4(x, ids, w64, L.codes, L.scales, L.gscales, shape.E,
                                             shape.H, shape.I, residual=residual, want_o=True,
                                             want_h=True)
    valid = (ids >= 0) & (ids < shape.E)
    assert_close_rms(h_g[valid], h_r[valid], what="nvfp4 h", max_ulps=h_ulps or ulps)
    assert_close_rms(o_g[valid], o_r[valid], what="nvfp4 o", max_ulps=ulps)
    if ulps > 1:
        # grouped products: the grouped paths' y rule (o-derived bound)
        check_grouped_y(y_g, y_r, o_g, o_r, w64, valid, residual, what="nvfp4 grouped y")
    else:
        assert_close_rms(y_g, y_r, what="nvfp4 y", max_ulps=2)
    for t in range(T):
        o_t = np.where(valid[t][:, None], o_g[t], 0).astype(np.uint16)
        want = oracle.combine(o_t, w64[t], None if residual is None else residual[t])
        np.testing.assert_array_equal(y_g[t], want)
    return y_g


@pytest.mark.parametrize("shape,T", [(synth.TINY, 1), (synth.TINY, 4), (synth.L24B, 1),
                                     (synth.L24B, 3), (synth.L8B, 4)])
def test_nvfp4_forward_matches_oracle(shape, T):
    L, layer = _layer(shape, 41)
    x = synth.make_tokens(T, shape.H, seed=41, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(41, 13, T))
    r = synth.make_tokens(T, shape.H, seed=42, stream=T) if T > 1 else None
    _check(L, layer, x, ids, w, shape, residual=r)
    assert layer.status() == 0
    layer.close()


# The grouped mma.sync products sum the exact products in another FP32
# order than the decode GEMVs; the tolerance is the MXFP4 grouped path's
# (reading R14: h and o within 2 BF16 values of the oracle).
@pytest.mark.parametrize("shape,T,dist,flags", [
    (synth.TINY, 11, "zipf", 0), (synth.TINY, 3, "uniform", moe.FWD_FORCE_MMA),
    (synth.L24B, 64, "uniform", 0), (synth.L24B, 64, "zipf", 0),
    (synth.L8B, 40, "uniform", moe.FWD_FORCE_GROUPED)])
def test_nvfp4_grouped_matches_oracle(shape, T, dist, flags):
    """Beyond 4 tokens (or forced) NVFP4 runs the grouped mma.sync products
    while the groups are small."""
    L, layer = _layer(shape, 43, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=43, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, dist, synth.rng_for(43, 13, T))
    r = synth.make_tokens(T, shape.H, seed=44, stream=T)
    _check(L, layer, x, ids, w, shape, residual=r, flags=flags, ulps=2)
    assert layer.status() == 0
    layer.close()


def _check_tcgen05_stages(L, layer, x, ids, w, shape, residual=None, flags=moe.FWD_FORCE_TCGEN05):
    """Stage by stage against the oracle (reading R14).  h: within 1e-2 rms of
    the oracle's h, except elements that the oracle's own rounding chain
    reproduces, h = BF16(BF16(silu(g')) u') , with g', u' and silu(g') each
    allowed one BF16 ulp away only where the exact value (FP64 from the
    oracle's dequantised rows) lies within 2^-16 of its accumulated magnitude
    of a rounding midpoint; such elements stay rare.  o: the oracle's down
    product of the kernel's own h (FP64, rounded once), within the decode
    tolerance.  y: bit-exact given the kernel's o, and within the o-derived
    bound of the oracle's y."""
    T = x.shape[0]
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=moe.FWD_KEEP_INTERMEDIATES | flags,
                      residual=None if residual is None else dev_bf16(residual))
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    _verify_stages(L, shape, x, ids, w, h_g, o_g, y_g, residual)
    return y_g


def _verify_stages(L, shape, x, ids, w, h_g, o_g, y_g, residual=None):
    """The checks of _check_tcgen05_stages on given kernel outputs (rows of
    a batch: x, ids, w, h, o, y of the same tokens)."""
    T = x.shape[0]
    w64 = w.astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward_nvfp4(x, ids, w64, L.codes, L.scales, L.gscales, shape.E,
                                             shape.H, shape.I, residual=residual, want_o=True,
                                             want_h=True)
    valid = (ids >= 0) & (ids < shape.E)
    matrix = lambda e, m: expert_matrix(L, shape, e, m, fmt="nvfp4")  # noqa: E731
    verify_h_flips(h_g, h_r, x, ids, valid, matrix, what="nvfp4 tcgen05 h")
    o_ref = o_given_h(h_g, ids, valid, matrix, shape.H)
    assert_close_rms(o_g[valid], o_ref[valid], what="nvfp4 tcgen05 o (given h)", max_ulps=2)
    check_grouped_y(y_g, y_r, o_g, o_r, w64, valid, residual, what="nvfp4 tcgen05 y", cap=False)
    for t in range(T):
        o_t = np.where(valid[t][:, None], o_g[t], 0).astype(np.uint16)
        want = oracle.combine(o_t, w64[t], None if residual is None else residual[t])
        np.testing.assert_array_equal(y_g[t], want)


@pytest.mark.parametrize("shape,T,dist", [
    (synth.L24B, 320, "uniform"), (synth.L24B, 260, "zipf"), (synth.L24B, 9, "uniform"),
    (synth.TINY, 100, "zipf"), (synth.TINY, 33, "uniform"), (synth.L8B, 40, "zipf")])
def test_nvfp4_tcgen05_matches_oracle(shape, T, dist):
    """NVFP4 on the tcgen05 products (A = E2M1 code x its block's E4M3 scale
    in BF16, exact; the expert's multiplier on the FP32 accumulator), stage
    by stage against the oracle; two runs give the same bits."""
    L, layer = _layer(shape, 49, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=49, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, dist, synth.rng_for(49, 13, T))
    r = synth.make_tokens(T, shape.H, seed=50, stream=T) if T % 2 else None
    y1 = _check_tcgen05_stages(L, layer, x, ids, w, shape, residual=r)
    y2 = _check_tcgen05_stages(L, layer, x, ids, w, shape, residual=r)
    np.testing.assert_array_equal(y1, y2)
    assert layer.status() == 0
    layer.close()


def test_nvfp4_tcgen05_chunks_and_automatic_choice():
    """2100 tokens of the 24B shape: the NVFP4 batch runs in launch sequences
    of 2048 tokens, the first on tcgen05 (its groups average 128 pairs per
    expert) and the ragged rest of 52 tokens on mma.sync.  Sampled tokens from
    both (h, o, y) against the oracle, stage by stage."""
    shape = synth.L24B
    T = 2100
    L, layer = _layer(shape, 51, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=51, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(51, 13, T))
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=moe.FWD_KEEP_INTERMEDIATES)
    torch.cuda.synchronize()
    assert layer.status() == 0
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    rows = np.r_[0:6, 2040:2056, 2094:2100]
    _verify_stages(L, shape, x[rows], ids[rows], w[rows], h_g[rows], o_g[rows], y_g[rows])
    layer.close()


def test_nvfp4_grouped_invalid_ids_and_decode_agreement():
    """Invalid ids on the grouped path zero the slot and flag; the forced
    per-(token, slot) path at the same T agrees with the grouped one within
    the tolerance and is deterministic."""
    shape = synth.L24B
    T = 9
    L, layer = _layer(shape, 48, max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=48)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(48, 13, T))
    ids[2, 1] = 99
    ids[7, 3] = -1
    y_g = _check(L, layer, x, ids, w, shape, ulps=2)
    assert layer.status() & moe.DEVICE_BAD_EXPERT_ID
    y_d = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_DECODE)
    y_d2 = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_DECODE)
    np.testing.assert_array_equal(y_d, y_d2)
    assert_close_rms(y_g, y_d, what="nvfp4 grouped vs decode y", max_ulps=2)
    layer.status()
    layer.close()


def test_nvfp4_invalid_ids_zero_the_slot_and_flag():
    shape = synth.TINY
    L, layer = _layer(shape, 44)
    x = synth.make_tokens(3, shape.H, seed=44)
    ids, w = synth.make_routing(3, shape.E, shape.top_k, "uniform", synth.rng_for(44, 13, 3))
    ids[1, 2] = 77
    ids[2, 0] = -5
    _check(L, layer, x, ids, w, shape)
    assert layer.status() & moe.DEVICE_BAD_EXPERT_ID
    layer.close()


def test_nvfp4_layer_is_route_then_forward():
    """moe_layer_ex on NVFP4 experts (every fusion setting runs the separate
    launches) gives the bits of moe_route_ex + moe_forward_ex."""
    shape = synth.L24B
    L, layer = _layer(shape, 45, bias=True)
    T = 2
    xr = dev_bf16(synth.make_tokens(T, shape.H, seed=45))
    res = dev_bf16(synth.make_tokens(T, shape.H, seed=46))
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
    y_r = oracle.moe_forward_nvfp4(xn_h, ids_h, w_h.astype(np.float64), L.codes, L.scales,
                                   L.gscales, shape.E, shape.H, shape.I,
                                   residual=host_bf16(res))
    assert_close_rms(y_h, y_r, what="nvfp4 layer y", max_ulps=2)
    layer.close()


def test_nvfp4_argument_errors():
    """H must suit the bulk-copy gate/up kernel (a multiple of 512); the
    multipliers are required."""
    shape = synth.LayerShape(E=4, H=256, I=128, top_k=2)
    L = synth.make_layer_nvfp4(shape, seed=47)
    h = moe.moe_create(shape.E, shape.H, shape.I, shape.top_k)
    try:
        with pytest.raises(moe.MoEError):
            moe.moe_load_packed_nvfp4(h, dev_u8(L.codes), dev_u8(L.scales),
                                      torch.from_numpy(L.gscales).cuda())
    finally:
        moe.moe_destroy(h)
