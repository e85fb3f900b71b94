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


def check_grouped_y(y_g, y_r, o_g, o_r, w64, valid, residual=None, what="grouped y", cap=True):
    """The grouped paths' rule for the combined output y (reading R14)."""
    # y is a function of o alone (the bit-exact combine check below), so its
    # distance to the oracle's y is bounded by the o differences through the
    # routing weights plus the two combines' own roundings (the kernel's and
    # the oracle's): k products, k sums and the residual add each, every one
    # off by at most half a BF16 ulp (<= 2^-8 of the value) of a value no
    # larger than the largest term, the result or the residual
    og, orr = f64(o_g), f64(o_r)
    og[~valid], orr[~valid] = 0.0, 0.0
    wa = np.abs(w64)[:, :, None]
    scale = np.maximum(np.abs(f64(y_r)), (wa * np.abs(orr)).max(axis=1))
    if residual is not None:
        scale = np.maximum(scale, np.abs(f64(residual)))
    k = w64.shape[1]
    bound = 1.01 * (wa * np.abs(og - orr)).sum(axis=1) + 2 * (2 * k + 1) * scale * 2.0 ** -8
    dy = np.abs(f64(y_g) - f64(y_r))
    assert np.all(dy <= bound), f"{what}: {(dy > bound).sum()} elements beyond the o-derived bound"
    # and a count limit on the elements beyond 1e-2 rms: an o flip under a
    # combine that cancels (|y| << |w o|) is many ulps of y, so the ulp
    # distance of those few elements is capped loosely but their number is
    # held to 0.05 % (observed worst: 7 of 65,536 at 2.8e-2 rms, 8 ulps, T=260
    # Zipf on tcgen05; all inside the o-derived bound above).  cap=False: the
    # caller verified o stage by stage (against the oracle's down product of
    # the kernel's own h), so only the derived bound applies here.
    if cap:
        assert_close_rms(y_g, y_r, what=what, max_ulps=16, max_flip_frac=5e-4)


# ---- stage-by-stage checks of the grouped products (reading R14) ----

def expert_matrix(L, shape, e, m, fmt="mxfp4"):
    """The oracle's dequantised matrix m (0 gate, 1 up, 2 down) of expert e,
    FP64 [rows, K]: MXFP4 (code x 2^(e-127)), NVFP4 (code x E4M3 block scale
    x the expert's multiplier) or sym8 (int8 x binary16 block scale)."""
    n = shape.I * shape.H
    rows, K = (shape.I, shape.H) if m < 2 else (shape.H, shape.I)
    if fmt == "sym8":
        q = np.ascontiguousarray(np.asarray(L.codes).reshape(shape.E, 3, n)[e, m])
        s = np.ascontiguousarray(np.asarray(L.scales).reshape(shape.E, 3, n // 32)[e, m])
        return oracle.dequant_sym8(q, s, n).reshape(rows, K)
    c = np.ascontiguousarray(L.codes.reshape(shape.E, 3, n // 2)[e, m])
    if fmt == "nvfp4":
        s = np.ascontiguousarray(L.scales.reshape(shape.E, 3, n // 16)[e, m])
        gs = float(L.gscales[e, 0 if m < 2 else 1])
        return oracle.dequant_nvfp4(c, s, gs, n).reshape(rows, K)
    s = np.ascontiguousarray(L.scales.reshape(shape.E, 3, n // 32)[e, m])
    return oracle.dequant(c, s, n).reshape(rows, K)


def _near_midpoint(v, mag, rel=2.0 ** -16):
    """v lies within rel * mag of a BF16 rounding midpoint (mag: the sum of
    the magnitudes an FP32 accumulation added, or |v| for one operation)."""
    b = oracle.bf16_from_f64(v)
    lo = oracle.bf16_to_f64(b)
    nb = oracle.bf16_to_f64(b + 1 if (v >= lo) == (v >= 0) else b - 1)
    return abs(v - (lo + nb) / 2) <= rel * mag


def _bf16_and_neighbours(v, movable):
    b = oracle.bf16_from_f64(v)
    vals = [oracle.bf16_to_f64(b)]
    if movable and b & 0x7FFF:
        vals += [oracle.bf16_to_f64(b + 1), oracle.bf16_to_f64(b - 1)]
    return vals


def verify_h_flips(h_g, h_r, x, ids, valid, matrix, what="h", max_frac=1e-3):
    """h of the grouped products against the oracle's h: every element beyond
    1e-2 rms must be the oracle's rounding chain h = BF16(BF16(silu(g')) u')
    with g', u' and silu(g') each allowed one BF16 ulp away only where that
    exact value (FP64, from the oracle's dequantised rows: matrix(e, m))
    lies within 2^-16 of its accumulated magnitude from a rounding midpoint;
    such elements stay below max_frac.  (With h = s u, two ulps of s can be
    four or more ulps of h, so an ulp count alone bounds nothing.)"""
    hg64, hr64 = f64(h_g), f64(h_r)
    rms = np.sqrt(np.mean(hr64 ** 2, axis=2, keepdims=True))
    far = valid[:, :, None] & (np.abs(hg64 - hr64) > TOL * rms)
    cache = {}
    for t, j, i in np.argwhere(far):
        e = int(ids[t, j])
        if e not in cache:
            cache = {e: (matrix(e, 0), matrix(e, 1))}
        wg, wu = cache[e][0][i], cache[e][1][i]
        xt = f64(x[t])
        g, u = float(wg @ xt), float(wu @ xt)
        g_ok = _near_midpoint(g, float(np.abs(wg * xt).sum()))
        u_ok = _near_midpoint(u, float(np.abs(wu * xt).sum()))
        want = float(hg64[t, j, i])
        hit = False
        for gg in _bf16_and_neighbours(g, g_ok):
            sl = gg / (1.0 + np.exp(-gg))
            for ss in _bf16_and_neighbours(sl, _near_midpoint(sl, abs(sl))):
                for uu in _bf16_and_neighbours(u, u_ok):
                    hit |= oracle.bf16_to_f64(oracle.bf16_from_f64(ss * uu)) == want
        assert hit, f"{what}[{t},{j},{i}] = {want} is no one-ulp rounding move of g={g}, u={u}"
    n = int(valid.sum()) * h_g.shape[2]
    print(f"[parity] {what}: {n} elements, {int(np.count_nonzero(hg64[valid] != hr64[valid]))} "
          f"differ, {int(far.sum())} beyond tol, each a one-ulp move of g, u or silu(g) at a "
          f"rounding midpoint")
    assert far.sum() <= max_frac * n, f"{what}: {far.sum()} elements beyond {TOL} rms"


def o_given_h(h_g, ids, valid, matrix, H):
    """The oracle's down product of the kernel's own h: o = BF16(W_down h) in
    FP64 per valid (token, slot), [T, k, H] BF16 bits (0 elsewhere)."""
    hg64 = f64(h_g)
    o_ref = np.zeros(h_g.shape[:2] + (H,), dtype=np.uint16)
    for e in np.unique(ids[valid]):
        wd = matrix(int(e), 2)
        sel = valid & (ids == e)
        o_ref[sel] = oracle.bf16_from_f64_array(hg64[sel] @ wd.T)
    return o_ref
