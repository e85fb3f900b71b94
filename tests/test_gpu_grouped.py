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
from gpu_util import assert_close_rms, dev_bf16, dev_layer, host_bf16
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
    # h = BF16(BF16(silu(BF16(g))) * BF16(u)): a one-ulp flip of g or u near a
    # rounding midpoint (different FP32 summation order on the tensor cores)
    # carries through silu and the product, so h (and o after it) may land two
    # BF16 values away; such flips stay rare (at most 1 % of the elements)
    assert_close_rms(h_g[valid], h_r[valid], what="grouped h", max_ulps=2)
    assert_close_rms(o_g[valid], o_r[valid], what="grouped o", max_ulps=2)
    # y is a function of o alone (the bit-exact combine check below); a
    # two-ulp flip of a large o term shows up in y as up to 4 of y's ulps when
    # the slot sum (and residual) partly cancel
    assert_close_rms(y_g, y_r, what="grouped y", max_ulps=4)
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


def test_grouped_more_tokens_than_one_launch_sequence():
    """T above the tokens of one grouped launch sequence runs in chunks."""
    shape = synth.TINY
    T = 300
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
