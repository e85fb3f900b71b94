"""CUDA-graph capture of the layer and of the stacked decode step: captured
and eager runs are bitwise equal, routing is recomputed on every replay, and
each layer of the stack matches the oracle fed that layer's GPU input."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, check_routing, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def test_layer_graph_replay_matches_eager_and_reroutes():
    shape = synth.L24B
    L = synth.make_layer(shape, seed=21)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, 4, codes, scales, rw, rb, max_tokens=1)
    x1 = synth.make_tokens(1, shape.H, seed=21, stream=1)
    x2 = synth.make_tokens(1, shape.H, seed=21, stream=2)
    xs = dev_bf16(x1)
    ids = torch.empty(1, 4, dtype=torch.int32, device="cuda")
    w = torch.empty(1, 4, dtype=torch.float32, device="cuda")
    y = torch.empty_like(xs)

    def run(stream=None):
        layer.route(xs, ids=ids, w=w, stream=stream)
        layer.forward(xs, ids, w, y=y, stream=stream)

    run()
    torch.cuda.synchronize()
    y_eager1, ids_eager1 = host_bf16(y).copy(), ids.cpu().numpy().copy()

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        run(s)
    y.zero_()
    g.replay()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(y), y_eager1)
    np.testing.assert_array_equal(ids.cpu().numpy(), ids_eager1)
    g.replay()  # repeated replay, same inputs -> same bits
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(y), y_eager1)

    # new input in place: the graph re-routes (selection is not frozen)
    xs.copy_(dev_bf16(x2))
    g.replay()
    torch.cuda.synchronize()
    ids_g2, y_g2 = ids.cpu().numpy().copy(), host_bf16(y).copy()
    rids, _, _ = oracle.route(x2, L.router_w, None, 4)
    assert not np.array_equal(rids, ids_eager1)
    run()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(ids_g2, ids.cpu().numpy())
    np.testing.assert_array_equal(y_g2, host_bf16(y))
    del g
    layer.close()


def _stack(shape, n_layers, seed, bias=False, T=1):
    layers = [synth.make_layer(shape, seed=seed, layer=l, bias=bias) for l in range(n_layers)]
    st = moe.MoEStack([dev_layer(L) for L in layers], shape.E, shape.H, shape.I, shape.top_k, T=T)
    return layers, st


@pytest.mark.parametrize("shape,n_layers,bias", [(synth.L24B, 4, False), (synth.L8B, 3, True),
                                                 (synth.TINY, 6, False)])
def test_stack_per_layer_parity_and_graph(shape, n_layers, bias):
    layers, st = _stack(shape, n_layers, seed=31, bias=bias)
    r0 = synth.make_tokens(1, shape.H, seed=31, stream=5)

    # eager, layer by layer, checking each against the oracle fed the GPU input
    st.r.copy_(dev_bf16(r0))
    logits = torch.empty(1, shape.E, dtype=torch.float32, device="cuda")
    for l, L in enumerate(layers):
        r_in = host_bf16(st.r).copy()
        lay = st.layers[l]
        moe.moe_route_ex(lay.handle, st.r, lay.router_w, lay.router_b, moe.ROUTE_RMSNORM, st.xn,
                         logits, st.ids[l], st.w[l])
        moe.moe_forward_ex(lay.handle, st.xn, st.ids[l], st.w[l], st.r, st.r, 0)
        torch.cuda.synchronize()
        xn_g = host_bf16(st.xn)
        xn_r = oracle.rmsnorm(r_in)
        assert_close_rms(xn_g, xn_r, tol=1e-2, what=f"rmsnorm layer {l}")
        rids, rw, rlg = oracle.route(xn_g, L.router_w, L.router_b, shape.top_k)
        check_routing(st.ids[l].cpu().numpy(), st.w[l].cpu().numpy(), logits.cpu().numpy(),
                      rids, rw, rlg, shape.top_k)
        ids_g = st.ids[l].cpu().numpy()
        w_g = st.w[l].cpu().numpy().astype(np.float64)
        r_out_ref = oracle.moe_forward(xn_g, ids_g, w_g, L.codes, L.scales, shape.E, shape.H,
                                       shape.I, residual=r_in)
        assert_close_rms(host_bf16(st.r), r_out_ref, what=f"layer {l} residual out", max_ulps=2)
    r_eager = host_bf16(st.r).copy()

    # the captured step replays to the same bits
    st.r.copy_(dev_bf16(r0))
    st.capture()
    st.r.copy_(dev_bf16(r0))
    st.step()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(st.r), r_eager)
    # a second step continues from the new residual (decode feedback)
    st.step()
    torch.cuda.synchronize()
    r2 = host_bf16(st.r).copy()
    st.graph = None
    st.r.copy_(dev_bf16(r_eager))
    st.enqueue()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(st.r), r2)
    st.close()
