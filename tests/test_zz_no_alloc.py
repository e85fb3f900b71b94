"""moe_forward_noalloc: the forward for callers that may not allocate device
memory (they run inside someone else's allocator or memory budget), checked
through the C ABI against the regular handle + workspace forward.

Collected last on purpose (file name), so a failure here leaves every other
test already run; it must also pass alone in a fresh process, where its first
call is the one that looks up the library's scratch array.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


def _call_raw(shape, codes, scales, x, ids, w, residual, y):
    lib = moe.load()
    p = lambda t: None if t is None else C.c_void_p(t.data_ptr())  # noqa: E731
    return lib.moe_forward_noalloc(
        shape.E, shape.H, shape.I, shape.top_k, p(codes), p(scales), p(x), x.shape[0], p(ids),
        p(w), p(residual), p(y), C.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("shape,T", [(synth.L24B, 1), (synth.TINY, 4)])
def test_noalloc_forward_matches_workspace_forward_twice(shape, T):
    L = synth.make_layer(shape, seed=41)
    codes, scales, rw, _ = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, None,
                         max_tokens=T)
    for call in range(2):  # two calls in a row, different tokens and routing
        x = dev_bf16(synth.make_tokens(T, shape.H, seed=41, stream=call))
        r = dev_bf16(synth.make_tokens(T, shape.H, seed=42, stream=call))
        ids_h, w_h = synth.make_routing(T, shape.E, shape.top_k, "uniform",
                                        synth.rng_for(41, call))
        ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
        ref = layer.forward(x, ids, w, residual=r)
        y = torch.empty_like(x)
        assert _call_raw(shape, codes, scales, x, ids, w, r, y) == 0
        torch.cuda.synchronize()
        assert_close_rms(host_bf16(y), host_bf16(ref), what=f"noalloc call {call}")
        # same kernels on the same inputs: identical bits
        np.testing.assert_array_equal(host_bf16(y), host_bf16(ref))
    layer.close()


def test_noalloc_rejects_sizes_beyond_its_scratch():
    shape = synth.L24B  # T * k * I * 2 bytes of h must fit the fixed scratch
    L = synth.make_layer(synth.TINY, seed=1)
    codes, scales = dev_layer(L)[:2]
    T = 64
    x = torch.zeros(T, shape.H, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(T, 4, dtype=torch.int32, device="cuda")
    w = torch.zeros(T, 4, dtype=torch.float32, device="cuda")
    y = torch.empty_like(x)
    assert _call_raw(shape, codes, scales, x, ids, w, None, y) == -5  # MOE_ERR_WORKSPACE


def test_noalloc_reports_a_bad_expert_id_through_its_status_word():
    """An id outside [0, E) zeroes that slot and sets MOE_DEVICE_BAD_EXPERT_ID
    in the scratch's status word, read (and cleared) by
    moe_forward_noalloc_status; the other slots still match the workspace
    forward given the same ids."""
    shape = synth.TINY
    T = 2
    L = synth.make_layer(shape, seed=43)
    codes, scales, rw, _ = dev_layer(L)
    layer = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, None,
                         max_tokens=T)
    x = dev_bf16(synth.make_tokens(T, shape.H, seed=43))
    ids_h, w_h = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(43, 1))
    assert moe.moe_forward_noalloc_status() == 0
    ids_h = ids_h.copy()
    ids_h[1, 2] = shape.E + 3
    ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
    y = torch.empty_like(x)
    moe.moe_forward_noalloc(shape.E, shape.H, shape.I, shape.top_k, codes, scales, x, ids, w,
                            None, y)
    assert moe.moe_forward_noalloc_status() & moe.DEVICE_BAD_EXPERT_ID
    assert moe.moe_forward_noalloc_status() == 0  # cleared by the read
    ref = layer.forward(x, ids, w)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host_bf16(y), host_bf16(ref))
    assert layer.status() & moe.DEVICE_BAD_EXPERT_ID
    layer.close()
