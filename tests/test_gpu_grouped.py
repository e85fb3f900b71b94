"""The (token, expert)-sorted grouped path (batches beyond the decode sizes)
against the oracle: SwiGLU vectors h, expert outputs o and combined y per
(token, slot), at the tolerance of the decode path; the combine bit-exact
given the kernel's own o; uniform and Zipf routing (many small groups, a few
large ones), ragged batch sizes, more tokens than one launch sequence takes,
invalid ids, and run-to-run determinism."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import (assert_close_rms, check_grouped_y, dev_bf16, dev_layer, expert_matrix,
                      host_bf16, o_given_h, verify_h_flips)
from workloads import synth

pytestmark = pytest.mark.gpu


def _setup(shape, seed, T, dist, max_tokens=None):
    L = synth.make_layer(shape, seed=seed)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                         max_tokens=max_tokens or T)
    x = synth.make_tokens(T, shape.H, seed=seed, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, dist, synth.rng_for(seed, 13, T))
    return L, layer, x, ids, w


def _check(L, layer, x, ids, w, shape, flags=0, residual=None):
    T = x.shape[0]
    xd = dev_bf16(x)
    y = layer.forward(xd, torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                      flags=flags | moe.FWD_KEEP_INTERMEDIATES,
                      residual=None if residual is None else dev_bf16(residual))
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    w64 = w.astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward(x, ids, w64, L.codes, L.scales, shape.E, shape.H,
                                       shape.I, residual=residual, want_o=True, want_h=True)
    valid = (ids >= 0) & (ids < shape.E)
    # h = BF16(BF16(silu(BF16(g))) * BF16(u)): the tensor-core tiles sum the
    # exact products in another FP32 order, so g or u near a BF16 rounding
    # midpoint may round the other way, and the flip carries through silu and
    # the product (several ulps of h when |u| is large).  Every h element
    # beyond 1e-2 rms must be such a one-ulp move at a midpoint, shown on the
    # exact FP64 values.  o is then checked against the oracle's down product
    # of the kernel's own h, so an h flip upstream does not count against it.
    matrix = lambda e, m: expert_matrix(L, shape, e, m)  # noqa: E731
    verify_h_flips(h_g, h_r, x, ids, valid, matrix, what="grouped h")
    o_ref = o_given_h(h_g, ids, valid, matrix, shape.H)
    assert_close_rms(o_g[valid], o_ref[valid], what="grouped o (given h)", max_ulps=2)
    check_grouped_y(y_g, y_r, o_g, o_r, w64, valid, residual, what="grouped y")
    # combine in slot order, bit-exact given the kernel's own expert outputs
    for t in range(T):
        o_t = np.where(valid[t][:, None], o_g[t], 0).astype(np.uint16)
        want = oracle.combine(o_t, w64[t], None if residual is None else residual[t])
        np.testing.assert_array_equal(y_g[t], want)
    return y_g


@pytest.mark.parametrize("shape,T,dist", [
    (synth.L24B, 5, "uniform"), (synth.L24B, 32, "uniform"), (synth.L24B, 32, "zipf"),
    (synth.L24B, 64, "zipf"), (synth.L8B, 17, "zipf"), (synth.TINY, 8, "uniform"),
    (synth.TINY, 33, "zipf"),
    # groups of 12 tokens on average: two 8-token chunks per CTA
    (synth.L24B, 200, "uniform"), (synth.TINY, 60, "uniform")])
def test_grouped_matches_oracle(shape, T, dist):
    L, layer, x, ids, w = _setup(shape, 71, T, dist)
    _check(L, layer, x, ids, w, shape)
    assert layer.status() == 0
    layer.close()


@pytest.mark.parametrize("shape,T,dist", [
    (synth.L24B, 320, "uniform"), (synth.L24B, 260, "zipf"), (synth.L24B, 9, "uniform"),
    (synth.TINY, 100, "zipf"), (synth.TINY, 33, "uniform")])
def test_grouped_tcgen05_matches_oracle(shape, T, dist):
    """The grouped products on tcgen05 (BF16 weight tiles, TMEM accumulators,
    TMA tensor loads of the packed codes): h, o, y against the oracle."""
    L, layer, x, ids, w = _setup(shape, 79, T, dist)
    _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_TCGEN05)
    assert layer.status() == 0
    layer.close()


def test_grouped_tcgen05_is_deterministic_and_needs_contiguous_weights():
    shape = synth.TINY
    L, layer, x, ids, w = _setup(shape, 80, 40, "zipf")
    y1 = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_TCGEN05)
    y2 = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_TCGEN05)
    np.testing.assert_array_equal(y1, y2)
    layer.close()
    # experts bound through a pointer table: no tensor map, the call is refused
    codes, scales, rw, rb = dev_layer(L)
    h = moe.moe_create(shape.E, shape.H, shape.I, shape.top_k)
    try:
        mc, ms = shape.I * shape.H // 2, shape.I * shape.H // 32
        cp = [codes.data_ptr() + (3 * e + m) * mc for e in range(shape.E) for m in range(3)]
        sp = [scales.data_ptr() + (3 * e + m) * ms for e in range(shape.E) for m in range(3)]
        moe.moe_load_expert_table(h, cp, sp)
        ws = torch.empty(moe.moe_workspace_bytes(h, 40), dtype=torch.uint8, device="cuda")
        moe.moe_set_workspace(h, ws, 40)
        y = torch.empty(40, shape.H, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(moe.MoEError):
            moe.moe_forward_ex(h, dev_bf16(x), torch.from_numpy(ids).cuda(),
                               torch.from_numpy(w).cuda(), None, y, moe.FWD_FORCE_TCGEN05)
    finally:
        moe.moe_destroy(h)


def test_grouped_tcgen05_wide_scale_span_rows():
    """Rows whose E8M0 exponents span 23, 24 and 30 binades (a group far
    below the row's largest): the BF16 weight tiles hold every code x scale
    exactly, so h, o, y still meet the oracle."""
    shape = synth.TINY
    T = 200
    L = synth.make_layer(shape, seed=82)
    H, I = shape.H, shape.I
    mat = I * H // 32  # scales of one matrix

    def put(e, m, r, g, v):
        K = H if m < 2 else I
        L.scales[e, m * mat + r * (K // 32) + g] = v

    hi = synth.E8M0_HI
    put(3, 0, 5, 0, hi)
    put(3, 0, 5, 1, hi - 30)        # gate row 5 of expert 3: span 30
    put(7, 2, 200, 0, hi)
    put(7, 2, 200, 2, hi - 24)      # down row 200 of expert 7: span 24
    put(5, 1, 70, 3, hi)
    put(5, 1, 70, 4, hi - 23)       # up row 70 of expert 5: span 23
    put(11, 2, 3, 0, hi)
    put(11, 2, 3, 1, hi - 23)       # down row 3 of expert 11: span 23
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                         max_tokens=T)
    x = synth.make_tokens(T, shape.H, seed=82)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(82, 13, T))
    for e in (3, 5, 7, 11):
        assert (ids == e).any()
    _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_TCGEN05)
    assert layer.status() == 0
    layer.close()


def test_grouped_residual_and_determinism():
    shape = synth.L24B
    L, layer, x, ids, w = _setup(shape, 72, 24, "zipf")
    r = synth.make_tokens(24, shape.H, seed=73)
    y1 = _check(L, layer, x, ids, w, shape, residual=r)
    y2 = _check(L, layer, x, ids, w, shape, residual=r)
    np.testing.assert_array_equal(y1, y2)
    layer.close()


def test_grouped_one_expert_takes_every_token():
    """Extreme skew: all tokens route to the same 4 experts (groups of T)."""
    shape = synth.TINY
    T = 70
    L, layer, x, _, w = _setup(shape, 74, T, "uniform")
    ids = np.tile(np.array([[3, 7, 0, 12]], dtype=np.int32), (T, 1))
    _check(L, layer, x, ids, w, shape)
    layer.close()


@pytest.mark.parametrize("T", [150])
def test_grouped_one_expert_group_beyond_one_pass(T):
    """Groups of T = 150 tokens: two token passes (128 + 22) of the tcgen05
    products (and 19 chunks of the mma.sync tiles)."""
    shape = synth.TINY
    L, layer, x, _, w = _setup(shape, 78, T, "uniform")
    ids = np.tile(np.array([[5, 2, 9, 14]], dtype=np.int32), (T, 1))
    y_mma = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_MMA)
    y_tc = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_TCGEN05)
    assert_close_rms(y_tc, y_mma, what="tcgen05 vs mma.sync", max_ulps=4)
    assert layer.status() == 0
    layer.close()


@pytest.mark.parametrize("shape", [synth.TINY, synth.L24B])
def test_grouped_product_choice_follows_group_size(shape):
    """Without a forcing flag the products run on tcgen05 exactly when the
    groups average at least 40 (token, slot) pairs (T k >= 40 E), else on the
    mma.sync tiles: the default call gives the bits of the forced one on each
    side of the threshold.  The two forcing flags exclude each other and the
    per-(token, slot) path."""
    t_min = 40 * shape.E // shape.top_k
    for T, forced in ((t_min, moe.FWD_FORCE_TCGEN05), (t_min - 1, moe.FWD_FORCE_MMA)):
        L, layer, x, ids, w = _setup(shape, 81, T, "zipf")
        args = (dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda())
        y0 = host_bf16(layer.forward(*args, flags=0)).copy()
        y1 = host_bf16(layer.forward(*args, flags=forced)).copy()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(y0, y1)
        assert layer.status() == 0
        for bad in (moe.FWD_FORCE_MMA | moe.FWD_FORCE_TCGEN05,
                    moe.FWD_FORCE_MMA | moe.FWD_FORCE_DECODE):
            with pytest.raises(moe.MoEError):
                layer.forward(*args, flags=bad)
        layer.close()


def test_grouped_more_tokens_than_one_launch_sequence():
    """T above the tokens of one grouped launch sequence runs in chunks."""
    shape = synth.TINY
    T = 2100
    L, layer, x, ids, w = _setup(shape, 75, T, "zipf")
    _check(L, layer, x, ids, w, shape)
    layer.close()


def test_grouped_invalid_ids_zero_the_slot_and_flag():
    shape = synth.TINY
    L, layer, x, ids, w = _setup(shape, 76, 9, "uniform")
    ids = ids.copy()
    ids[2, 1] = 99
    ids[5, 3] = -1
    _check(L, layer, x, ids, w, shape)
    st = layer.status()
    assert st & moe.DEVICE_BAD_EXPERT_ID
    layer.close()


@pytest.mark.parametrize("T", [1, 3])
def test_forced_grouped_small_batch_matches_decode(T):
    """FORCE_GROUPED at decode sizes: the oracle's result, and the decode
    path's within the same tolerance (different accumulation order)."""
    shape = synth.L24B
    L, layer, x, ids, w = _setup(shape, 77, T, "uniform", max_tokens=4)
    y_g = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_GROUPED)
    y_d = _check(L, layer, x, ids, w, shape, flags=moe.FWD_FORCE_DECODE)
    assert_close_rms(y_g, y_d, what="grouped vs decode", max_ulps=2)
    layer.close()


def test_tcgen05_two_layers_alternating_keep_their_tensor_maps():
    """Two handles bound to different weights, their tcgen05 forwards
    interleaved: each handle encodes its own tensor maps, so every call gives
    the bits of the same handle's first call."""
    shape = synth.TINY
    T = 100
    a = _setup(shape, 81, T, "uniform")
    b = _setup(shape, 82, T, "uniform")
    flags = moe.FWD_FORCE_TCGEN05
    firsts = []
    for L, layer, x, ids, w in (a, b):
        y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(),
                          flags=flags)
        torch.cuda.synchronize()
        firsts.append(host_bf16(y).copy())
    for _ in range(3):
        for i, (L, layer, x, ids, w) in enumerate((a, b)):
            y = layer.forward(dev_bf16(x), torch.from_numpy(ids).cuda(),
                              torch.from_numpy(w).cuda(), flags=flags)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(host_bf16(y), firsts[i])
    _check(*a[:5], shape, flags=flags)
    for t in (a, b):
        t[1].close()


def test_status_read_on_one_stream():
    """moe_get_status_stream reads (and clears) the status of the work queued
    on the given stream."""
    shape = synth.TINY
    L, layer, x, ids, w = _setup(shape, 83, 9, "uniform")
    ids = ids.copy()
    ids[4, 0] = 200
    s = torch.cuda.Stream()
    xd, idd, wd = dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        layer.forward(xd, idd, wd, stream=s)
    assert layer.status(stream=s) & moe.DEVICE_BAD_EXPERT_ID
    assert layer.status(stream=s) == 0  # cleared
    layer.close()
