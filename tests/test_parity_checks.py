"""Pins of the grouped path's stage-by-stage parity checks (tests/gpu_util.py:
verify_h_flips, o_given_h), on the CPU with the oracle's own outputs standing
in for a kernel's.  The checks must pass the oracle itself, catch a planted
error in h or o, accept an h whose g rounded to the other BF16 neighbour where
the exact g lies at a rounding midpoint, and reject the same move where g
lies far from one."""
import numpy as np
import pytest

import oracle
from gpu_util import TOL, assert_close_rms, expert_matrix, f64, o_given_h, verify_h_flips
from workloads import synth

FORMATS = {
    "mxfp4": (synth.make_layer, lambda L, s, x, ids, w: oracle.moe_forward(
        x, ids, w, L.codes, L.scales, s.E, s.H, s.I, want_o=True, want_h=True)),
    "nvfp4": (synth.make_layer_nvfp4, lambda L, s, x, ids, w: oracle.moe_forward_nvfp4(
        x, ids, w, L.codes, L.scales, L.gscales, s.E, s.H, s.I, want_o=True, want_h=True)),
    "sym8": (synth.make_layer_sym8, lambda L, s, x, ids, w: oracle.moe_forward_sym8(
        x, ids, w, L.codes, L.scales, s.E, s.H, s.I, want_o=True, want_h=True)),
}


def _case(fmt, T=12, seed=91):
    shape = synth.TINY
    make, fwd = FORMATS[fmt]
    L = make(shape, seed=seed)
    x = synth.make_tokens(T, shape.H, seed=seed, stream=T)
    ids, w = synth.make_routing(T, shape.E, shape.top_k, "uniform", synth.rng_for(seed, 13, T))
    y, o, h = fwd(L, shape, x, ids, w.astype(np.float64))
    valid = (ids >= 0) & (ids < shape.E)
    matrix = lambda e, m: expert_matrix(L, shape, e, m, fmt=fmt)  # noqa: E731
    return shape, x, ids, valid, matrix, o, h


def _bf16(v):
    return oracle.bf16_to_f64(oracle.bf16_from_f64(v))


def _other_neighbour(g):
    """The BF16 neighbour of g on the other side of the rounding decision."""
    b = oracle.bf16_from_f64(g)
    lo = oracle.bf16_to_f64(b)
    return oracle.bf16_to_f64(b + 1 if (g >= lo) == (g >= 0) else b - 1)


def _gu_all(shape, x, ids, valid, matrix):
    """Exact g, u, sum |w x| of every valid (token, slot, row)."""
    out = []
    for e in np.unique(ids[valid]):
        wg, wu = matrix(int(e), 0), matrix(int(e), 1)
        for t, j in np.argwhere(valid & (ids == e)):
            xt = f64(x[t])
            g, u = wg @ xt, wu @ xt
            mag = np.abs(wg * xt).sum(axis=1)
            for i in range(shape.I):
                out.append((t, j, i, float(g[i]), float(u[i]), float(mag[i])))
    return out


@pytest.mark.parametrize("fmt", list(FORMATS))
def test_stage_checks_pass_the_oracle_itself(fmt):
    shape, x, ids, valid, matrix, o, h = _case(fmt)
    verify_h_flips(h, h, x, ids, valid, matrix, what=f"{fmt} h (oracle)")
    np.testing.assert_array_equal(o_given_h(h, ids, valid, matrix, shape.H)[valid], o[valid])


@pytest.mark.parametrize("fmt", list(FORMATS))
def test_stage_checks_catch_planted_errors(fmt):
    shape, x, ids, valid, matrix, o, h = _case(fmt)
    t, j = np.argwhere(valid)[3]
    hb = h.copy()
    hb[t, j, 5] = oracle.bf16_from_f64(f64(np.array([h[t, j, 5]]))[0] * 1.1 + 0.3)
    with pytest.raises(AssertionError):
        verify_h_flips(hb, h, x, ids, valid, matrix, what="planted h")
    ob = o.copy()
    ob[t, j, 9] = oracle.bf16_from_f64(f64(np.array([o[t, j, 9]]))[0] + 4.0)
    with pytest.raises(AssertionError):
        assert_close_rms(ob[valid], o_given_h(h, ids, valid, matrix, shape.H)[valid],
                         what="planted o", max_ulps=2)


def test_one_ulp_move_of_g_is_accepted_only_at_a_midpoint():
    shape, x, ids, valid, matrix, o, h = _case("mxfp4", T=24)
    hr64 = f64(h)
    rms = np.sqrt(np.mean(hr64 ** 2, axis=2))
    near = far = None
    for t, j, i, g, u, mag in _gu_all(shape, x, ids, valid, matrix):
        moved = oracle.bf16_from_f64(_other_neighbour(g) / (1.0 + np.exp(-_other_neighbour(g))))
        h2 = oracle.bf16_from_f64(oracle.bf16_to_f64(moved) * _bf16(u))
        if abs(oracle.bf16_to_f64(h2) - hr64[t, j, i]) <= TOL * rms[t, j]:
            continue  # the move stays within the tolerance: nothing to decide
        b = oracle.bf16_from_f64(g)
        gap = abs(g - (oracle.bf16_to_f64(b) + _other_neighbour(g)) / 2)
        if near is None and gap <= 2.0 ** -18 * mag:
            near = (t, j, i, h2)
        if far is None and gap >= 0.25 * abs(_other_neighbour(g) - oracle.bf16_to_f64(b)):
            far = (t, j, i, h2)
        if near and far:
            break
    assert near is not None and far is not None
    for (t, j, i, h2), ok in ((near, True), (far, False)):
        hb = h.copy()
        hb[t, j, i] = h2
        if ok:
            verify_h_flips(hb, h, x, ids, valid, matrix, what="g moved at a midpoint")
        else:
            with pytest.raises(AssertionError):
                verify_h_flips(hb, h, x, ids, valid, matrix, what="g moved far from a midpoint")
