"""Helpers shared by the GPU parity tests: move seeded inputs to the device,
bring results back as BF16 bits, and the comparison rules."""
import numpy as np
import torch

import oracle

TOL = 1e-2  # max|gpu - oracle| <= TOL * rms(oracle), per output vector


def dev_bf16(u16: np.ndarray) -> torch.Tensor:
    a = np.ascontiguousarray(u16, dtype=np.uint16)
    return torch.from_numpy(a.view(np.int16)).cuda().view(torch.bfloat16)


def host_bf16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def dev_u8(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.uint8)).cuda()


def dev_layer(L):
    """workloads.LayerInputs -> device tensors (codes, scales, router_w, router_b)."""
    rb = None if L.router_b is None else torch.from_numpy(L.router_b).cuda()
    return dev_u8(L.codes), dev_u8(L.scales), dev_bf16(L.router_w), rb


def f64(u16):
    return oracle.bf16_to_f64_array(u16)


def ulp_distance(a_u16, b_u16):
    """Number of BF16 values between a and b (0 = equal, 1 = adjacent)."""
    def ordinal(u):
        u = np.asarray(u, dtype=np.int64)
        return np.where(u & 0x8000, -(u & 0x7FFF), u)
    return np.abs(ordinal(a_u16) - ordinal(b_u16))


def assert_close_rms(gpu_u16, ref_u16, tol=TOL, what="", max_ulps=1, max_flip_frac=0.01):
    """Per vector (last axis): every element within tol * rms(ref) of the
    oracle, except rounding flips: elements where the GPU (FP32 accumulation)
    and the oracle (FP64) land on BF16 values at most `max_ulps` apart because
    the exact value sits near a BF16 rounding midpoint.  One BF16 ulp exceeds
    1e-2 * rms for any element above ~1.28 * rms, so such flips are allowed,
    counted, and must stay rare (<= max_flip_frac of the elements).
    Returns (flips, elements that differ at all)."""
    gpu_u16 = np.asarray(gpu_u16).reshape(-1, np.shape(ref_u16)[-1])
    ref_u16 = np.asarray(ref_u16).reshape(gpu_u16.shape)
    g, r = f64(gpu_u16), f64(ref_u16)
    assert np.all(np.isfinite(g)) and np.all(np.isfinite(r)), what
    rms = np.sqrt(np.mean(r * r, axis=1, keepdims=True))
    err = np.abs(g - r)
    within = err <= tol * rms
    ulps = ulp_distance(gpu_u16, ref_u16)
    flip = (~within) & (ulps <= max_ulps)
    bad = (~within) & ~flip
    worst = int(ulps.max()) if ulps.size else 0
    if what:
        # observed distances, so that any loosening of a rule shows in the log
        print(f"[parity] {what}: {gpu_u16.size} elements, {int(np.count_nonzero(g != r))} "
              f"differ, {int(flip.sum())} rounding flips beyond tol, worst {worst} ulp, "
              f"max err {float((err / rms).max()):.2e} x rms")
    assert not np.any(bad), (f"{what}: {bad.sum()} elements beyond tolerance, worst "
                             f"{(err / rms)[bad].max():.3e} x rms, {ulps[bad].max()} ulps")
    assert flip.mean() <= max_flip_frac, f"{what}: flip fraction {flip.mean():.4f}"
    return int(flip.sum()), int(np.count_nonzero(g != r))


def near_tie_tokens(logits: np.ndarray, k: int, rel=1e-4):
    """Tokens whose oracle logits leave a gap < rel*max|logit| between any two
    of the k+1 largest (the selection or the slot order could flip under a
    different summation order)."""
    flags = []
    for row in np.atleast_2d(logits):
        s = np.sort(row)[::-1][: k + 1]
        gaps = s[:-1] - s[1:]
        flags.append(bool(np.min(gaps) < rel * np.max(np.abs(row))))
    return np.array(flags)


def check_routing(gpu_ids, gpu_w, gpu_logits, ref_ids, ref_w, ref_logits, k):
    """Ids bit-exact to the oracle except on flagged near-ties, where they must
    equal the oracle's selector applied to the GPU's own logits.  Weights
    within 1e-5 relative.  Returns the number of near-tie tokens."""
    ties = near_tie_tokens(ref_logits, k)
    np.testing.assert_allclose(gpu_logits, ref_logits, rtol=1e-4, atol=1e-4)
    for t in range(gpu_ids.shape[0]):
        if ties[t]:
            ids2, w2 = oracle.select_topk(gpu_logits[t].astype(np.float64), k)
            np.testing.assert_array_equal(gpu_ids[t], ids2[0])
            np.testing.assert_allclose(gpu_w[t], w2[0], rtol=1e-5, atol=1e-6)
        else:
            np.testing.assert_array_equal(gpu_ids[t], ref_ids[t])
            np.testing.assert_allclose(gpu_w[t], ref_w[t], rtol=1e-5, atol=1e-6)
    return int(ties.sum())
