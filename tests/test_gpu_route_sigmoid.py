"""Sigmoid scoring of the router (MOE_ROUTE_SIGMOID) on the GPU against the
oracle: unbiased logits, top-k of sigmoid(l) + bias, coefficients from the
selected unbiased scores; and the whole layer with that scoring."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu

WIDE = synth.LayerShape(E=160, H=256, I=64, top_k=8)  # E > 64: the wide top-k


def _keys(logits, bias):
    s = 1.0 / (1.0 + np.exp(-np.asarray(logits, dtype=np.float64)))
    return s + (0.0 if bias is None else np.asarray(bias, dtype=np.float64))


def _near_ties(keys, k, rel=1e-5):
    """Tokens whose k + 1 largest keys come closer than rel * max|key|: the
    selection or its order may legitimately differ between FP32 and FP64."""
    out = []
    for row in np.atleast_2d(keys):
        s = np.sort(row)[::-1][: k + 1]
        out.append(bool(np.min(s[:-1] - s[1:]) < rel * np.max(np.abs(row))))
    return np.array(out)


def _check(gpu_ids, gpu_w, gpu_lg, x, L, k):
    rids, rw, rlg = oracle.route(x, L.router_w, L.router_b, k, sigmoid=True)
    # the logits stay unbiased
    np.testing.assert_allclose(gpu_lg, rlg, rtol=1e-4, atol=1e-4)
    ties = _near_ties(_keys(rlg, L.router_b), k)
    for t in range(gpu_ids.shape[0]):
        if ties[t]:
            # the oracle's selector on the GPU's own logits
            ids2, w2 = oracle.select_topk_sigmoid(gpu_lg[t].astype(np.float64), L.router_b, k)
            np.testing.assert_array_equal(gpu_ids[t], ids2[0])
            np.testing.assert_allclose(gpu_w[t], w2[0], rtol=1e-5, atol=1e-6)
        else:
            np.testing.assert_array_equal(gpu_ids[t], rids[t])
            np.testing.assert_allclose(gpu_w[t], rw[t], rtol=1e-5, atol=1e-6)
    return rids, rw


@pytest.mark.parametrize("shape,T,bias", [(synth.TINY, 4, False), (synth.TINY, 4, True),
                                          (synth.L24B, 1, True), (synth.L8B, 3, True),
                                          (synth.L24B, 40, True), (WIDE, 5, True)])
def test_sigmoid_route_matches_oracle(shape, T, bias):
    for seed in range(3):
        L = synth.make_layer(shape, seed=seed, bias=bias)
        x = synth.make_tokens(T, shape.H, seed=seed, stream=T)
        codes, scales, rw, rb = dev_layer(L)
        layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                             max_tokens=max(T, 4))
        lg = torch.empty(T, shape.E, dtype=torch.float32, device="cuda")
        ids, w = layer.route(dev_bf16(x), logits=lg, sigmoid=True)
        torch.cuda.synchronize()
        g_ids, g_w = ids.cpu().numpy(), w.cpu().numpy()
        _check(g_ids, g_w, lg.cpu().numpy(), x, L, shape.top_k)
        np.testing.assert_allclose(g_w.sum(axis=1), 1.0, rtol=1e-5)
        layer.close()


def test_sigmoid_bias_steers_selection_only():
    """A large bias on one expert puts it first for every token, while its
    coefficient stays its unbiased score over the selected scores."""
    shape = synth.L24B
    L = synth.make_layer(shape, seed=21)
    L.router_b = np.zeros(shape.E, dtype=np.float32)
    L.router_b[37] = 10.0
    x = synth.make_tokens(4, shape.H, seed=21)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb)
    lg = torch.empty(4, shape.E, dtype=torch.float32, device="cuda")
    ids, w = layer.route(dev_bf16(x), logits=lg, sigmoid=True)
    torch.cuda.synchronize()
    g_ids, g_w = ids.cpu().numpy(), w.cpu().numpy()
    assert np.all(g_ids[:, 0] == 37)
    _check(g_ids, g_w, lg.cpu().numpy(), x, L, shape.top_k)
    layer.close()


@pytest.mark.parametrize("shape,T", [(synth.L24B, 1), (synth.L8B, 4), (synth.TINY, 3)])
def test_sigmoid_layer_is_route_then_forward(shape, T):
    """moe_layer_ex with sigmoid scoring (and the RMSNorm) gives the bits of
    moe_route_ex + moe_forward_ex, and the oracle's layer within tolerance."""
    L = synth.make_layer(shape, seed=31, bias=True)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                         max_tokens=4)
    xr = synth.make_tokens(T, shape.H, seed=31, stream=T)
    res = synth.make_tokens(T, shape.H, seed=32, stream=T)
    flags = moe.ROUTE_SIGMOID | moe.ROUTE_RMSNORM
    outs = []
    for fused in (True, False):
        xn = torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda")
        lg = torch.zeros(T, shape.E, dtype=torch.float32, device="cuda")
        ids = torch.zeros(T, shape.top_k, dtype=torch.int32, device="cuda")
        w = torch.zeros(T, shape.top_k, dtype=torch.float32, device="cuda")
        y = torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda")
        if fused:
            moe.moe_layer_ex(layer.handle, dev_bf16(xr), layer.router_w, layer.router_b, flags,
                             xn, lg, ids, w, dev_bf16(res), y, 0)
        else:
            moe.moe_route_ex(layer.handle, dev_bf16(xr), layer.router_w, layer.router_b, flags,
                             xn, lg, ids, w)
            moe.moe_forward_ex(layer.handle, xn, ids, w, dev_bf16(res), y, 0)
        torch.cuda.synchronize()
        outs.append((host_bf16(xn).copy(), lg.cpu().numpy(), ids.cpu().numpy(),
                     w.cpu().numpy(), host_bf16(y).copy()))
        assert layer.status() == 0
    for a, b in zip(outs[0], outs[1]):
        np.testing.assert_array_equal(a, b)
    xn, lg, g_ids, g_w, y = outs[0]
    _check(g_ids, g_w, lg, xn, L, shape.top_k)
    y_r = oracle.moe_forward(xn, g_ids, g_w.astype(np.float64), L.codes, L.scales, shape.E,
                             shape.H, shape.I, residual=res)
    assert_close_rms(y, y_r, what="sigmoid layer y", max_ulps=2)
    layer.close()
