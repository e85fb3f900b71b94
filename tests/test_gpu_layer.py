"""moe_layer_ex in its three launch structures -- the whole layer in one
launch, the router inside the gate/up launch (logits exchanged between CTAs and
the routing handed to the down launch through tagged workspace words), and
separate launches -- against each other and against moe_route_ex +
moe_forward_ex, bit for bit, and against the oracle."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, check_routing, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _bufs(T, shape):
    return dict(
        xn=torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda"),
        logits=torch.zeros(T, shape.E, dtype=torch.float32, device="cuda"),
        ids=torch.zeros(T, shape.top_k, dtype=torch.int32, device="cuda"),
        w=torch.zeros(T, shape.top_k, dtype=torch.float32, device="cuda"),
        y=torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda"),
    )


def _layer_ex(layer, x, b, rmsnorm, residual):
    moe.moe_layer_ex(layer.handle, x, layer.router_w, layer.router_b,
                     moe.ROUTE_RMSNORM if rmsnorm else 0, b["xn"] if rmsnorm else None,
                     b["logits"], b["ids"], b["w"], residual, b["y"], 0)


def _split(layer, x, b, rmsnorm, residual):
    moe.moe_route_ex(layer.handle, x, layer.router_w, layer.router_b,
                     moe.ROUTE_RMSNORM if rmsnorm else 0, b["xn"] if rmsnorm else None,
                     b["logits"], b["ids"], b["w"])
    moe.moe_forward_ex(layer.handle, b["xn"] if rmsnorm else x, b["ids"], b["w"], residual,
                       b["y"], 0)


def _host(b):
    return {k: (host_bf16(v) if v.dtype == torch.bfloat16 else v.cpu().numpy()).copy()
            for k, v in b.items()}


@pytest.mark.parametrize("shape,T,bias,rmsnorm", [
    (synth.L24B, 1, False, True), (synth.L24B, 2, False, True), (synth.L24B, 4, True, False),
    (synth.L8B, 3, True, True), (synth.TINY, 1, False, False), (synth.TINY, 4, True, True)])
def test_fused_layer_bitwise_equals_unfused_and_split(shape, T, bias, rmsnorm):
    """Every launch structure gives the same bits (the one-launch layer falls
    back to two launches where its shared memory plan does not fit)."""
    L = synth.make_layer(shape, seed=51, bias=bias)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                         max_tokens=4)
    # several calls in a row on one workspace: the routing handoff counters
    # advance once per call and must stay in step across fused / unfused calls
    for call in range(4):
        x = dev_bf16(synth.make_tokens(T, shape.H, seed=51, stream=call))
        res = dev_bf16(synth.make_tokens(T, shape.H, seed=52, stream=call)) if call % 2 else None
        outs = {}
        modes = {"layer": moe.FUSION_LAYER, "fused": moe.FUSION_ROUTER,
                 "unfused": moe.FUSION_NONE, "split": None}
        for mode, fusion in modes.items():
            b = _bufs(T, shape)
            if fusion is not None:
                moe.moe_set_fusion(layer.handle, fusion)
            (_split if fusion is None else _layer_ex)(layer, x, b, rmsnorm, res)
            torch.cuda.synchronize()
            outs[mode] = _host(b)
            assert layer.status() == 0, mode
        for mode in ("fused", "unfused", "split"):
            for key in ("xn", "logits", "ids", "w", "y"):
                np.testing.assert_array_equal(outs["layer"][key], outs[mode][key],
                                              err_msg=f"{key}: one launch vs {mode}, call {call}")
        # and the result is the oracle's layer (routing checked with near-tie care)
        xr = host_bf16(x)
        xn_r = oracle.rmsnorm(xr) if rmsnorm else xr
        if rmsnorm:
            assert_close_rms(outs["fused"]["xn"], xn_r, tol=1e-2, what="x_norm")
        xin = outs["fused"]["xn"] if rmsnorm else xr
        rids, rw_, rlg = oracle.route(xin, L.router_w, L.router_b, shape.top_k)
        check_routing(outs["fused"]["ids"], outs["fused"]["w"], outs["fused"]["logits"],
                      rids, rw_, rlg, shape.top_k)
        y_r = oracle.moe_forward(xin, outs["fused"]["ids"],
                                 outs["fused"]["w"].astype(np.float64), L.codes, L.scales,
                                 shape.E, shape.H, shape.I,
                                 residual=None if res is None else host_bf16(res))
        assert_close_rms(outs["fused"]["y"], y_r, what=f"fused y, call {call}", max_ulps=2)
    layer.close()


@pytest.mark.parametrize("fusion", [1, 2])
def test_fused_layer_in_graph_with_shared_workspace(fusion):
    """A captured stack of fused layers sharing one workspace replays to the
    eager bits, replay after replay (the per-call tags keep advancing)."""
    shape = synth.L24B
    layers = [synth.make_layer(shape, seed=61, layer=l) for l in range(3)]
    st = moe.MoEStack([dev_layer(L) for L in layers], shape.E, shape.H, shape.I, shape.top_k,
                      persistent=False)
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=61, stream=1))
    want = {}
    for mode in (moe.FUSION_NONE, fusion):  # the fused stack matches the unfused one
        st.set_fusion(mode)
        st.r.copy_(r0)
        st.enqueue()
        torch.cuda.synchronize()
        r1 = host_bf16(st.r).copy()
        st.enqueue()
        torch.cuda.synchronize()
        want[mode] = (r1, host_bf16(st.r).copy())
    np.testing.assert_array_equal(want[fusion][0], want[moe.FUSION_NONE][0])
    np.testing.assert_array_equal(want[fusion][1], want[moe.FUSION_NONE][1])
    r1, r2 = want[fusion]
    st.r.copy_(r0)
    st.capture()
    for want in (r1, r2):
        st.step()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_bf16(st.r), want)
    for L in st.layers:
        assert L.status() == 0
    st.close()
