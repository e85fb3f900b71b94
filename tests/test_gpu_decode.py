"""GPU parity of the decode path (C-ABI through the thin binding) against the
CPU oracle, on the same seeded inputs."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import (assert_close_rms, check_routing, dev_bf16, dev_layer, dev_u8, host_bf16)
from workloads import synth

pytestmark = pytest.mark.gpu


def make(shape, seed, T, bias=False, max_tokens=None):
    L = synth.make_layer(shape, seed=seed, bias=bias)
    x = synth.make_tokens(T, shape.H, seed=seed, stream=T)
    codes, scales, rw, rb = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, rb,
                         max_tokens=max_tokens or max(T, 4))
    return L, x, layer


# ----------------------------------------------------------- dequant ------

def test_dequant_exhaustive_bitwise():
    """All 256 byte values x all 256 E8M0 exponents through the kernels' own
    in-register decode, bitwise against the oracle (FP32)."""
    codes = np.tile(np.arange(256, dtype=np.uint8), 256)
    scales = np.repeat(np.arange(256, dtype=np.uint8), 16)
    n = codes.size * 2
    out = torch.empty(n, dtype=torch.float32, device="cuda")
    moe.moe_debug_dequant(dev_u8(codes), dev_u8(scales), n, out)
    got = out.cpu().numpy()
    want = oracle.dequant_f32(codes, scales, n)
    nan = np.isnan(want)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), want[~nan].view(np.uint32))


# ------------------------------------------------------------- route -------

@pytest.mark.parametrize("shape,T,bias", [(synth.TINY, 4, False), (synth.L24B, 1, False),
                                          (synth.L24B, 4, True), (synth.L8B, 3, True)])
def test_route_matches_oracle(shape, T, bias):
    for seed in range(3):
        L, x, layer = make(shape, seed, T, bias=bias)
        xd = dev_bf16(x)
        logits = torch.empty(T, shape.E, dtype=torch.float32, device="cuda")
        ids = torch.empty(T, shape.top_k, dtype=torch.int32, device="cuda")
        w = torch.empty(T, shape.top_k, dtype=torch.float32, device="cuda")
        layer.route(xd, ids=ids, w=w, logits=logits)
        torch.cuda.synchronize()
        rids, rw, rlg = oracle.route(x, L.router_w, L.router_b, shape.top_k)
        check_routing(ids.cpu().numpy(), w.cpu().numpy(), logits.cpu().numpy(), rids, rw, rlg,
                      shape.top_k)
        layer.close()


def test_route_ties_go_to_lower_id():
    """Identical router rows give equal logits: the lower expert id wins."""
    shape = synth.LayerShape(E=16, H=256, I=64, top_k=4)
    L = synth.make_layer(shape, seed=9)
    rw = L.router_w.copy()
    rw[5] = rw[2]
    rw[11] = rw[2]
    x = synth.make_tokens(1, shape.H, seed=9)
    # make row 2 the best by construction: align it with x
    rw[2] = x[0]
    rw[5] = x[0]
    rw[11] = x[0]
    codes, scales, _, _ = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, 4, codes, scales, dev_bf16(rw), None)
    ids, w = layer.route(dev_bf16(x))
    assert ids.cpu().numpy()[0, :3].tolist() == [2, 5, 11]
    rids, _, _ = oracle.route(x, rw, None, 4)
    assert ids.cpu().numpy().tolist() == rids.tolist()
    layer.close()


# ----------------------------------------------------------- forward -------

def _forward_checks(L, x, layer, ids, w, T, shape):
    xd = dev_bf16(x)
    y = layer.forward(xd, ids, w, flags=moe.FWD_KEEP_INTERMEDIATES)
    torch.cuda.synchronize()
    h_g, o_g = layer.intermediates(T)
    h_g, o_g, y_g = host_bf16(h_g), host_bf16(o_g), host_bf16(y)
    ids_h = ids.cpu().numpy()
    w_h = w.cpu().numpy().astype(np.float64)
    y_r, o_r, h_r = oracle.moe_forward(x, ids_h, w_h, L.codes, L.scales, shape.E, shape.H,
                                       shape.I, want_o=True, want_h=True)
    assert_close_rms(h_g, h_r, what="h")
    assert_close_rms(o_g, o_r, what="o")
    assert_close_rms(y_g, y_r, what="y", max_ulps=2)
    # the combine is bit-exact given the kernel's own expert outputs
    for t in range(T):
        np.testing.assert_array_equal(y_g[t], oracle.combine(o_g[t], w_h[t]))
    return y_g


@pytest.mark.parametrize("shape,T", [(synth.TINY, 4), (synth.TINY, 1), (synth.TINY, 3),
                                     (synth.L24B, 1), (synth.L24B, 2), (synth.L8B, 1)])
def test_forward_matches_oracle(shape, T):
    for seed in range(2):
        L, x, layer = make(shape, seed, T)
        rng = synth.rng_for(seed, 7, T)
        ids_h, w_h = synth.make_routing(T, shape.E, shape.top_k, "uniform", rng)
        ids = torch.from_numpy(ids_h).cuda()
        w = torch.from_numpy(w_h).cuda()
        _forward_checks(L, x, layer, ids, w, T, shape)
        assert layer.status() == 0
        layer.close()


@pytest.mark.parametrize("shape,T", [(synth.TINY, 4), (synth.L24B, 1), (synth.L8B, 2)])
def test_layer_end_to_end(shape, T):
    """route + forward on the GPU vs oracle.moe_layer (same seeded inputs)."""
    bias = shape is synth.L8B
    for seed in range(3):
        L, x, layer = make(shape, seed, T, bias=bias)
        xd = dev_bf16(x)
        logits = torch.empty(T, shape.E, dtype=torch.float32, device="cuda")
        ids, w = layer.route(xd, logits=logits)
        y = layer.forward(xd, ids, w)
        torch.cuda.synchronize()
        rids, rw, rlg = oracle.route(x, L.router_w, L.router_b, shape.top_k)
        ids_g, w_g = ids.cpu().numpy(), w.cpu().numpy()
        ties = check_routing(ids_g, w_g, logits.cpu().numpy(), rids, rw, rlg, shape.top_k)
        if ties:
            # a near-tie token may legitimately pick other experts (the GPU's
            # own selection was checked above): its y is compared with the
            # oracle's forward under the GPU's routing, the others' with the
            # oracle's whole layer
            print(f"[parity] layer y seed {seed}: {ties} near-tie token(s) of {T}")
        _, _, y_r = oracle.moe_layer(x, L.router_w, L.router_b, L.codes, L.scales, shape.E,
                                     shape.H, shape.I, shape.top_k)
        y_own = oracle.moe_forward(x, ids_g, w_g.astype(np.float64), L.codes, L.scales, shape.E,
                                   shape.H, shape.I)
        same = np.all(ids_g == rids, axis=1)
        y_ref = np.where(same[:, None], y_r, y_own)
        assert_close_rms(host_bf16(y), y_ref, what="layer y", max_ulps=2)
        layer.close()


@pytest.mark.parametrize("E,H,I,k,T", [(8, 96, 160, 8, 2), (1, 64, 64, 1, 1), (5, 64, 32, 5, 3),
                                       (12, 2880, 2880, 4, 1), (16, 512, 384, 2, 4)])
def test_edge_shapes(E, H, I, k, T):
    """Ragged chunk counts (K/32 not a multiple of the team size), k = E,
    a single expert, wide rows."""
    shape = synth.LayerShape(E=E, H=H, I=I, top_k=k)
    L, x, layer = make(shape, 5, T)
    rng = synth.rng_for(5, 8)
    ids_h = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    w_h = rng.random((T, k)).astype(np.float32)
    _forward_checks(L, x, layer, torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda(),
                    T, shape)
    layer.close()


def test_tokens_beyond_decode_chunk():
    """T = 7 on a workspace for 8 tokens (decode path runs in token chunks)."""
    shape = synth.TINY
    L, x, layer = make(shape, 3, 7, max_tokens=8)
    rng = synth.rng_for(3, 9)
    ids_h, w_h = synth.make_routing(7, shape.E, 4, "zipf", rng)
    _forward_checks(L, x, layer, torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda(),
                    7, shape)
    layer.close()


@pytest.mark.parametrize("shape", [synth.TINY, synth.L24B])
def test_invalid_ids_zero_the_slot_and_flag(shape):
    """TINY streams down rows from global memory, L24B copies them into shared
    memory first (rows of an invalid id are not fetched there)."""
    L, x, layer = make(shape, 4, 2)
    ids_h = np.array([[3, 99, 5, -1], [0, 1, 2, 3]], dtype=np.int32)
    w_h = np.array([[0.4, 0.3, 0.2, 0.1], [0.25] * 4], dtype=np.float32)
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda())
    st = layer.status()
    assert st & moe.DEVICE_BAD_EXPERT_ID
    assert layer.status() == 0  # cleared by the read
    y_r = oracle.moe_forward(x, ids_h, w_h.astype(np.float64), L.codes, L.scales, shape.E,
                             shape.H, shape.I)
    assert_close_rms(host_bf16(y), y_r, what="y with invalid ids", max_ulps=2)
    layer.close()


def test_tuning_switches_do_not_change_results():
    shape = synth.L24B
    L, x, layer = make(shape, 6, 1)
    xd = dev_bf16(x)
    ids, w = layer.route(xd)
    outs = []
    for pdl, pf in ((True, True), (False, False), (True, False), (False, True)):
        moe.moe_set_tuning(layer.handle, pdl, pf)
        outs.append(host_bf16(layer.forward(xd, ids, w)))
    for o in outs[1:]:
        np.testing.assert_array_equal(o, outs[0])
    layer.close()


def test_residual_fused_add():
    shape = synth.TINY
    L, x, layer = make(shape, 8, 2)
    r = synth.make_tokens(2, shape.H, seed=99)
    rng = synth.rng_for(8, 3)
    ids_h, w_h = synth.make_routing(2, shape.E, 4, "uniform", rng)
    rd = dev_bf16(r)
    y = layer.forward(dev_bf16(x), torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda(),
                      y=rd, residual=rd)  # in place
    y_r = oracle.moe_forward(x, ids_h, w_h.astype(np.float64), L.codes, L.scales, shape.E,
                             shape.H, shape.I, residual=r)
    assert_close_rms(host_bf16(y), y_r, what="residual y", max_ulps=2)
    layer.close()


def test_argument_errors_from_host():
    shape = synth.TINY
    L, x, layer = make(shape, 1, 1)
    xd = dev_bf16(x)
    ids = torch.zeros(1, 4, dtype=torch.int32, device="cuda")
    w = torch.zeros(1, 4, dtype=torch.float32, device="cuda")
    y = torch.empty_like(xd)
    lib = moe.load()
    import ctypes as C
    h = C.c_void_p(layer.handle)
    s = C.c_void_p(torch.cuda.current_stream().cuda_stream)
    # host pointer instead of device memory
    host = np.zeros(shape.H, dtype=np.uint16)
    assert lib.moe_forward(h, C.c_void_p(host.ctypes.data), 1, C.c_void_p(ids.data_ptr()),
                           C.c_void_p(w.data_ptr()), C.c_void_p(y.data_ptr()), s) == -3
    # misaligned
    assert lib.moe_forward(h, C.c_void_p(xd.data_ptr() + 2), 1, C.c_void_p(ids.data_ptr()),
                           C.c_void_p(w.data_ptr()), C.c_void_p(y.data_ptr()), s) == -4
    # T beyond the workspace
    assert lib.moe_forward(h, C.c_void_p(xd.data_ptr()), 5, C.c_void_p(ids.data_ptr()),
                           C.c_void_p(w.data_ptr()), C.c_void_p(y.data_ptr()), s) == -5
    # y aliasing x
    assert lib.moe_forward(h, C.c_void_p(xd.data_ptr()), 1, C.c_void_p(ids.data_ptr()),
                           C.c_void_p(w.data_ptr()), C.c_void_p(xd.data_ptr()), s) == -1
    with pytest.raises(moe.MoEError):
        moe.moe_forward(layer.handle, xd.float(), ids, w, y)
    layer.close()
