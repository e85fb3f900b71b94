"""The whole decode step of a stack of layers in one persistent launch
(moe_stack_*): every layer against the oracle fed that layer's GPU input
(RMSNorm, routing with near-tie handling, expert FFN + combine + residual),
bit-for-bit against the same stack run one layer at a time, under CUDA-graph
capture and decode feedback, with experts bound through scattered pointer
tables, and a bounded wait that gives up (reported, and the next step runs
normally)."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, check_routing, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _layers(shape, n_layers, seed, bias=False):
    return [synth.make_layer(shape, seed=seed, layer=l, bias=bias) for l in range(n_layers)]


def _hist(shape, n):
    dev = "cuda"
    return dict(r_hist=torch.zeros(n, shape.H, dtype=torch.bfloat16, device=dev),
                xn_hist=torch.zeros(n, shape.H, dtype=torch.bfloat16, device=dev),
                logits=torch.zeros(n, shape.E, dtype=torch.float32, device=dev),
                topk_ids=torch.zeros(n, shape.top_k, dtype=torch.int32, device=dev),
                topk_w=torch.zeros(n, shape.top_k, dtype=torch.float32, device=dev))


def _check_layers_against_oracle(shape, layers, hist, r_out, nvfp4=False):
    """Layer l: xn = RMSNorm(r_in) and the routing of xn against the oracle;
    the layer output (next layer's input, or the final r) against the
    oracle's expert FFN + combine + residual fed the GPU's xn and routing
    (nvfp4: the oracle's NVFP4 experts)."""
    n = len(layers)
    r_hist = host_bf16(hist["r_hist"])
    xn_hist = host_bf16(hist["xn_hist"])
    logits = hist["logits"].cpu().numpy()
    ids = hist["topk_ids"].cpu().numpy()
    w = hist["topk_w"].cpu().numpy()
    ties = 0
    for l, L in enumerate(layers):
        xn_r = oracle.rmsnorm(r_hist[l:l + 1])
        assert_close_rms(xn_hist[l:l + 1], xn_r, what=f"rmsnorm layer {l}")
        rids, rw, rlg = oracle.route(xn_hist[l:l + 1], L.router_w, L.router_b, shape.top_k)
        ties += check_routing(ids[l:l + 1], w[l:l + 1], logits[l:l + 1], rids, rw, rlg, shape.top_k)
        w64 = w[l:l + 1].astype(np.float64)
        if nvfp4:
            out_ref = oracle.moe_forward_nvfp4(xn_hist[l:l + 1], ids[l:l + 1], w64, L.codes,
                                               L.scales, L.gscales, shape.E, shape.H, shape.I,
                                               residual=r_hist[l:l + 1])
        else:
            out_ref = oracle.moe_forward(xn_hist[l:l + 1], ids[l:l + 1], w64, L.codes, L.scales,
                                         shape.E, shape.H, shape.I, residual=r_hist[l:l + 1])
        out_gpu = r_hist[l + 1:l + 2] if l + 1 < n else r_out
        assert_close_rms(out_gpu, out_ref, what=f"layer {l} output", max_ulps=2)
    return ties


@pytest.mark.parametrize("shape,n_layers,bias", [(synth.L24B, 5, False), (synth.L8B, 4, True),
                                                 (synth.TINY, 7, False)])
def test_stack_kernel_matches_oracle_and_layer_path(shape, n_layers, bias):
    layers = _layers(shape, n_layers, seed=61, bias=bias)
    st = moe.MoEStack([dev_layer(L) for L in layers], shape.E, shape.H, shape.I, shape.top_k)
    assert st.stack is not None
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=61, stream=3))

    # reference: the same step one layer at a time
    st.r.copy_(r0)
    st.enqueue_layers()
    torch.cuda.synchronize()
    r_layers = host_bf16(st.r).copy()
    ids_layers = st.ids.cpu().numpy().copy()

    # one launch, with every layer's intermediates kept
    hist = _hist(shape, n_layers)
    st.r.copy_(r0)
    moe.moe_stack_decode(st.stack, st.r, **hist)
    torch.cuda.synchronize()
    assert st.status() == 0
    r_stack = host_bf16(st.r).copy()
    np.testing.assert_array_equal(r_stack, r_layers)
    np.testing.assert_array_equal(hist["topk_ids"].cpu().numpy(), ids_layers.reshape(n_layers, -1))
    np.testing.assert_array_equal(host_bf16(hist["r_hist"][0:1]), host_bf16(r0))
    _check_layers_against_oracle(shape, layers, hist, r_stack)

    # captured: replays give the eager bits; a second step continues from the
    # first one's output (decode feedback)
    st.r.copy_(r0)
    st.capture()
    st.r.copy_(r0)
    st.step()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(st.r), r_stack)
    st.step()
    torch.cuda.synchronize()
    r2 = host_bf16(st.r).copy()
    st.graph = None
    st.r.copy_(dev_bf16(r_stack))
    st.enqueue_layers()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(st.r), r2)
    assert st.status() == 0
    st.close()


@pytest.mark.parametrize("shape,n_layers,bias", [(synth.L24B, 4, False), (synth.TINY, 5, False),
                                                 (synth.L8B, 3, True)])
def test_stack_kernel_nvfp4_matches_oracle_and_layer_path(shape, n_layers, bias):
    """NVFP4 experts (an E4M3 scale per 16 elements, FP32 multipliers per
    expert) in the one-launch stack: bit-for-bit the same step run one layer
    at a time (route + NVFP4 gate/up + down kernels), every layer within the
    oracle's tolerance (NVFP4 expert FFN fed the GPU's routed vector and
    routing), and a graph replay gives the eager bits."""
    layers = [synth.make_layer_nvfp4(shape, seed=63, layer=l, bias=bias) for l in range(n_layers)]
    w = [dev_layer(L) + (torch.from_numpy(L.gscales).cuda(),) for L in layers]
    st = moe.MoEStack(w, shape.E, shape.H, shape.I, shape.top_k)
    assert st.stack is not None
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=63, stream=3))
    st.r.copy_(r0)
    st.enqueue_layers()
    torch.cuda.synchronize()
    r_layers = host_bf16(st.r).copy()
    ids_layers = st.ids.cpu().numpy().copy()
    hist = _hist(shape, n_layers)
    st.r.copy_(r0)
    moe.moe_stack_decode(st.stack, st.r, **hist)
    torch.cuda.synchronize()
    assert st.status() == 0
    r_stack = host_bf16(st.r).copy()
    np.testing.assert_array_equal(r_stack, r_layers)
    np.testing.assert_array_equal(hist["topk_ids"].cpu().numpy(), ids_layers.reshape(n_layers, -1))
    _check_layers_against_oracle(shape, layers, hist, r_stack, nvfp4=True)
    st.r.copy_(r0)
    st.capture()
    st.r.copy_(r0)
    st.step()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(st.r), r_stack)
    assert st.status() == 0
    st.close()


def test_stack_many_steps_stay_bitwise_with_the_layer_path():
    """Twenty decode steps of a 3-layer 24B stack, graph-replayed: after each
    step the residual equals the layer-by-layer path's (launch counter and
    tags advance across launches)."""
    shape = synth.L24B
    layers = _layers(shape, 3, seed=62)
    w = [dev_layer(L) for L in layers]
    st = moe.MoEStack(w, shape.E, shape.H, shape.I, shape.top_k)
    ref = moe.MoEStack(w, shape.E, shape.H, shape.I, shape.top_k, persistent=False)
    assert st.stack is not None and ref.stack is None
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=62, stream=1))
    st.r.copy_(r0)
    ref.r.copy_(r0)
    st.capture()
    st.r.copy_(r0)
    for _ in range(20):
        st.step()
        ref.enqueue()
        torch.cuda.synchronize()
        np.testing.assert_array_equal(host_bf16(st.r), host_bf16(ref.r))
    assert st.status() == 0
    st.close()
    ref.close()


def test_stack_with_scattered_expert_tables():
    """Layers whose experts are bound through moe_load_expert_table at
    scattered addresses (permuted order, inside a larger pool) give the bits
    of the contiguously bound stack."""
    shape = synth.L24B
    layers = _layers(shape, 2, seed=63)
    w = [dev_layer(L) for L in layers]
    st_c = moe.MoEStack(w, shape.E, shape.H, shape.I, shape.top_k)
    mc, ms = shape.I * shape.H // 2, shape.I * shape.H // 32
    g = np.random.default_rng(63)
    pools, handles = [], []
    for (codes, scales, rw, rb) in w:
        slots = g.permutation(3 * shape.E + 5)  # a pool with spare slots
        cpool = torch.zeros((3 * shape.E + 5) * mc, dtype=torch.uint8, device="cuda")
        spool = torch.zeros((3 * shape.E + 5) * ms, dtype=torch.uint8, device="cuda")
        cflat, sflat = codes.view(-1), scales.view(-1)
        cp, sp = [], []
        for i in range(3 * shape.E):
            s_ = int(slots[i])
            cpool[s_ * mc:(s_ + 1) * mc] = cflat[i * mc:(i + 1) * mc]
            spool[s_ * ms:(s_ + 1) * ms] = sflat[i * ms:(i + 1) * ms]
            cp.append(cpool.data_ptr() + s_ * mc)
            sp.append(spool.data_ptr() + s_ * ms)
        h = moe.moe_create(shape.E, shape.H, shape.I, shape.top_k)
        moe.moe_load_expert_table(h, cp, sp)
        ws = torch.empty(moe.moe_workspace_bytes(h, 1), dtype=torch.uint8, device="cuda")
        moe.moe_set_workspace(h, ws, 1)
        pools.append((cpool, spool, ws))
        handles.append(h)
    s = moe.moe_stack_create(handles, [x[2] for x in w], [x[3] for x in w])
    sws = torch.empty(moe.moe_stack_workspace_bytes(s), dtype=torch.uint8, device="cuda")
    moe.moe_stack_set_workspace(s, sws)
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=63, stream=2))
    r_t = r0.clone()
    moe.moe_stack_decode(s, r_t)
    st_c.r.copy_(r0)
    st_c.enqueue()
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(r_t), host_bf16(st_c.r))
    assert moe.moe_stack_get_status(s) == 0
    moe.moe_stack_destroy(s)
    for h in handles:
        moe.moe_destroy(h)
    st_c.close()


def test_stack_wait_that_gives_up_is_reported_and_the_next_step_runs():
    """With the tagged-word waits limited to zero polls the first wait on
    another CTA gives up: the step sets MOE_DEVICE_TIMEOUT, leaves r as it
    was (no layer output is written), drains its own copies and exits; the
    context stays usable and the next step (normal limit) gives the reference
    bits."""
    shape = synth.L24B
    layers = _layers(shape, 2, seed=64)
    st = moe.MoEStack([dev_layer(L) for L in layers], shape.E, shape.H, shape.I, shape.top_k)
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=64, stream=4))
    st.r.copy_(r0)
    st.enqueue_layers()
    torch.cuda.synchronize()
    want = host_bf16(st.r).copy()
    st.r.copy_(r0)
    moe.moe_stack_set_spin_limit(st.stack, 0)
    st.enqueue()
    assert moe.moe_stack_get_status(st.stack) & moe.DEVICE_TIMEOUT
    np.testing.assert_array_equal(host_bf16(st.r), host_bf16(r0))
    moe.moe_stack_set_spin_limit(st.stack, 1 << 20)
    st.enqueue()
    assert moe.moe_stack_get_status(st.stack) == 0
    np.testing.assert_array_equal(host_bf16(st.r), want)
    st.close()


def test_stack_refuses_what_it_does_not_hold():
    """A stack mixing MXFP4 and NVFP4 layers, and several tokens per step,
    run one layer at a time (moe_stack_create refuses the mixed stack)."""
    shape = synth.L24B
    L = synth.make_layer_nvfp4(shape, seed=65)
    Lm = synth.make_layer(shape, seed=65)
    codes, scales = torch.from_numpy(L.codes).cuda(), torch.from_numpy(L.scales).cuda()
    gs = torch.from_numpy(L.gscales).cuda()
    rw = dev_bf16(L.router_w)
    st = moe.MoEStack([dev_layer(Lm), (codes, scales, rw, None, gs)], shape.E, shape.H, shape.I,
                      shape.top_k)
    assert st.stack is None
    with pytest.raises(moe.MoEError):
        moe.moe_stack_create([x.handle for x in st.layers], [x.router_w for x in st.layers])
    st.close()
    st2 = moe.MoEStack([dev_layer(Lm)], shape.E, shape.H, shape.I, shape.top_k, T=2)
    assert st2.stack is None
    st2.close()
