"""Experts bound through the device expert-pointer table (moe_load_expert_table,
model card section "Direct reads from GPU-resident weights"): every matrix
sits at its own address inside a larger pool, in permuted order, so the kernels
must read the table (no base address arithmetic can find them).  The decode
path (T = 1 and 4), the grouped mma.sync path (T = 64, Zipf routing) and every
launch structure of a whole layer are compared with the oracle and bit for bit
with the same layer bound contiguously."""
import numpy as np
import pytest
import torch

import oracle
import packed_mxfp4_w4a16_b200 as moe
from gpu_util import assert_close_rms, dev_bf16, dev_layer, host_bf16
from workloads import synth

pytestmark = pytest.mark.gpu


class TableLayer:
    """A handle whose 3E matrices are copied into a pool of 3E + 7 slots in a
    seeded permuted order and bound with moe_load_expert_table."""

    def __init__(self, shape, L, seed, max_tokens):
        codes, scales, _, _ = dev_layer(L)
        mc, ms = shape.I * shape.H // 2, shape.I * shape.H // 32
        n = 3 * shape.E
        slots = np.random.default_rng(seed).permutation(n + 7)
        self.cpool = torch.zeros((n + 7) * mc, dtype=torch.uint8, device="cuda")
        self.spool = torch.zeros((n + 7) * ms, dtype=torch.uint8, device="cuda")
        cflat, sflat = codes.view(-1), scales.view(-1)
        cp, sp = [], []
        for i in range(n):
            s_ = int(slots[i])
            self.cpool[s_ * mc:(s_ + 1) * mc] = cflat[i * mc:(i + 1) * mc]
            self.spool[s_ * ms:(s_ + 1) * ms] = sflat[i * ms:(i + 1) * ms]
            cp.append(self.cpool.data_ptr() + s_ * mc)
            sp.append(self.spool.data_ptr() + s_ * ms)
        self.handle = moe.moe_create(shape.E, shape.H, shape.I, shape.top_k)
        moe.moe_load_expert_table(self.handle, cp, sp)
        self.ws = torch.empty(moe.moe_workspace_bytes(self.handle, max_tokens),
                              dtype=torch.uint8, device="cuda")
        moe.moe_set_workspace(self.handle, self.ws, max_tokens)

    def forward(self, x, ids, w, flags=0):
        y = torch.empty_like(x)
        moe.moe_forward_ex(self.handle, x, ids, w, None, y, flags)
        return y

    def close(self):
        moe.moe_destroy(self.handle)


@pytest.mark.parametrize("shape,T,dist,flags", [
    (synth.L24B, 1, "uniform", 0), (synth.TINY, 4, "uniform", 0),
    (synth.L24B, 4, "zipf", moe.FWD_FORCE_DECODE),
    (synth.L24B, 64, "zipf", moe.FWD_FORCE_MMA), (synth.TINY, 40, "uniform", 0)])
def test_table_bound_experts_match_oracle_and_contiguous(shape, T, dist, flags):
    L = synth.make_layer(shape, seed=51)
    codes, scales, rw, _ = dev_layer(L)
    cont = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, None,
                        max_tokens=T)
    tab = TableLayer(shape, L, seed=52, max_tokens=T)
    x_h = synth.make_tokens(T, shape.H, seed=51, stream=T)
    ids_h, w_h = synth.make_routing(T, shape.E, shape.top_k, dist, synth.rng_for(51, 3, T))
    x = dev_bf16(x_h)
    ids, w = torch.from_numpy(ids_h).cuda(), torch.from_numpy(w_h).cuda()
    y_t = host_bf16(tab.forward(x, ids, w, flags))
    y_c = host_bf16(cont.forward(x, ids, w, flags=flags))
    torch.cuda.synchronize()
    np.testing.assert_array_equal(y_t, y_c)
    y_r = oracle.moe_forward(x_h, ids_h, w_h.astype(np.float64), L.codes, L.scales, shape.E,
                             shape.H, shape.I)
    assert_close_rms(y_t, y_r, what=f"table-bound y T={T}", max_ulps=2)
    assert moe.moe_get_status(tab.handle) == 0
    tab.close()
    cont.close()


@pytest.mark.parametrize("fusion", [moe.FUSION_NONE, moe.FUSION_ROUTER, moe.FUSION_LAYER])
def test_table_bound_layer_in_every_launch_structure(fusion):
    """moe_layer_ex (RMSNorm, routing inside the expert kernels, residual) on
    table-bound experts equals the contiguous layer bit for bit."""
    shape = synth.L24B
    L = synth.make_layer(shape, seed=53)
    codes, scales, rw, _ = dev_layer(L)
    cont = moe.MoELayer(shape.E, shape.H, shape.I, shape.top_k, codes, scales, rw, None,
                        max_tokens=1)
    tab = TableLayer(shape, L, seed=54, max_tokens=1)
    for h in (cont.handle, tab.handle):
        moe.moe_set_fusion(h, fusion)
    r0 = dev_bf16(synth.make_tokens(1, shape.H, seed=53, stream=2))
    outs = []
    for h in (cont.handle, tab.handle):
        r = r0.clone()
        xn = torch.empty_like(r)
        ids = torch.zeros(1, shape.top_k, dtype=torch.int32, device="cuda")
        w = torch.zeros(1, shape.top_k, dtype=torch.float32, device="cuda")
        moe.moe_layer_ex(h, r, rw, None, moe.ROUTE_RMSNORM, xn, None, ids, w, r, r, 0)
        torch.cuda.synchronize()
        outs.append((host_bf16(r).copy(), ids.cpu().numpy().copy()))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    assert moe.moe_get_status(tab.handle) == 0
    tab.close()
    cont.close()
