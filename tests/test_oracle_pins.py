"""Pins of the CPU oracle against facts that do not come from the oracle.

Each test checks an oracle function against something independent of it:
the E2M1 bit-field definition and the value table printed for the format,
powers of two, hand-derived BF16 roundings and combine sequences (fixtures
under tests/golden/, each with its citation), binary32 rounding done by
torch, dense brute force with an independently written unpacker, stable
library sorting and softmax, and the closed forms of the model arithmetic.
"""
import math

import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from workloads import synth

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


# ------------------------------------------------------------ helpers (test)

def e2m1_bitfield(code):
    """E2M1 from its bit fields: sign (bit 3), exponent (bits 2..1, bias 1),
    mantissa (bit 0); exponent field 0 is subnormal (0.5 * mantissa)."""
    s = (code >> 3) & 1
    E = (code >> 1) & 3
    m = code & 1
    mag = 0.5 * m if E == 0 else 2.0 ** (E - 1) * (1.0 + 0.5 * m)
    return -mag if s else mag


def unpack_dense(codes_m, scales_m, rows, K):
    """Independent unpacker: packed [rows][K/2] + E8M0 [rows][K/32] -> f64."""
    b = np.asarray(codes_m, dtype=np.uint8).reshape(rows, K // 2)
    nib = np.empty((rows, K), dtype=np.int64)
    nib[:, 0::2] = b & 0x0F
    nib[:, 1::2] = b >> 4
    table = np.array([e2m1_bitfield(c) for c in range(16)])
    v = table[nib]
    e = np.asarray(scales_m, dtype=np.float64).reshape(rows, K // 32)
    sc = np.repeat(np.exp2(e - 127.0), 32, axis=1)
    return v * sc


def bf16_via_f32(v):
    """BF16 bits of float64 values, rounded through binary32 by torch."""
    t = torch.from_numpy(np.asarray(v, dtype=np.float64)).to(torch.float32)
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_f64(b):
    return oracle.bf16_to_f64_array(b)


def ulp_diff(a, b):
    """Distance in BF16 ulps between two arrays of BF16 bits (same sign)."""
    ai = np.asarray(a, dtype=np.int32)
    bi = np.asarray(b, dtype=np.int32)
    ai = np.where(ai & 0x8000, 0x8000 - ai, ai)
    bi = np.where(bi & 0x8000, 0x8000 - bi, bi)
    return np.abs(ai - bi)


# --------------------------------------------------------------- E2M1/E8M0

def test_e2m1_matches_printed_table(golden):
    for row in golden("e2m1_values.txt"):
        code, val = row.split()
        v = oracle.e2m1_value(int(code))
        assert v == float(val)
        assert math.copysign(1.0, v) == math.copysign(1.0, float(val))


def test_e2m1_matches_bitfield_definition():
    for c in range(16):
        assert oracle.e2m1_value(c) == e2m1_bitfield(c)


def test_e8m0_powers_of_two():
    assert oracle.e8m0_value(127) == 1.0
    assert oracle.e8m0_value(0) == 2.0 ** -127
    assert oracle.e8m0_value(254) == 2.0 ** 127
    assert math.isnan(oracle.e8m0_value(255))
    for e in range(254):
        assert oracle.e8m0_value(e + 1) == 2.0 * oracle.e8m0_value(e)


def test_dequant_exhaustive_all_bytes_all_exponents():
    # every byte value in every position parity, with every exponent
    bytes_row = np.arange(256, dtype=np.uint8)              # 512 elements
    codes = np.tile(bytes_row, 256)
    scales = np.repeat(np.arange(256, dtype=np.uint8), 16)  # 16 groups/row
    n = 512 * 256
    got = oracle.dequant(codes, scales, n).reshape(256, 512)
    table = np.array([e2m1_bitfield(c) for c in range(16)])
    lo = table[bytes_row & 0x0F]
    hi = table[bytes_row >> 4]
    row = np.empty(512)
    row[0::2], row[1::2] = lo, hi
    for e in range(256):
        sc = math.ldexp(1.0, e - 127) if e != 255 else float("nan")
        exp = row * sc
        if e == 255:
            assert np.all(np.isnan(got[e]))
        else:
            np.testing.assert_array_equal(got[e], exp)
            assert np.array_equal(np.signbit(got[e]), np.signbit(exp))


def test_dequant_group_indexing():
    # constant code 2 (= 1.0), one distinct exponent per 32-element group
    K = 32 * 8
    codes = np.full(K // 2, 0x22, dtype=np.uint8)
    scales = np.arange(120, 128, dtype=np.uint8)
    got = oracle.dequant(codes, scales, K)
    exp = np.repeat(2.0 ** (scales.astype(float) - 127), 32)
    np.testing.assert_array_equal(got, exp)


def test_dequant_f32_matches_binary32_cast():
    # every code with every finite exponent; overflow (>= 2^128) must give inf
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8), 2)
    table = np.array([e2m1_bitfield(c) for c in range(16)])
    for e in range(255):
        got = oracle.dequant_f32(codes, np.array([e], dtype=np.uint8), 32)
        want = (np.tile(table, 2) * math.ldexp(1.0, e - 127)).astype(np.float32)
        np.testing.assert_array_equal(got, want)
    got = oracle.dequant_f32(codes, np.array([254], dtype=np.uint8), 32)
    assert np.isinf(got[7]) and got[3] == np.float32(1.5 * 2.0 ** 127)


# ------------------------------------------------------------------- BF16

def test_bf16_golden_roundings(golden):
    for row in golden("bf16_rounding.txt"):
        expr, hexv, _why = [s.strip() for s in row.split("|")]
        v = float(eval(expr, {"__builtins__": {}}, {}))
        assert oracle.bf16_from_f64(v) == int(hexv, 16), expr


def test_bf16_matches_binary32_routine():
    rng = np.random.default_rng(7)
    bits = rng.integers(0, 2 ** 32, size=200_000, dtype=np.uint64).astype(np.uint32)
    f = bits.view(np.float32)
    f = f[np.isfinite(f)]
    # plus exact ties and subnormals
    ties = ((rng.integers(0, 2 ** 15, 5000).astype(np.uint32) << 16) | 0x8000).view(np.float32)
    sub = (rng.integers(1, 2 ** 23, 5000).astype(np.uint32)).view(np.float32)
    f = np.concatenate([f, ties[np.isfinite(ties)], sub])
    want = torch.from_numpy(f.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = oracle.bf16_from_f64_array(f.astype(np.float64))
    np.testing.assert_array_equal(got, want)


def test_bf16_to_double_roundtrip():
    b = np.arange(0, 2 ** 16, dtype=np.uint32).astype(np.uint16)
    v = bf16_f64(b)
    finite = np.isfinite(v)
    back = oracle.bf16_from_f64_array(v[finite])
    # -0 and +0 both round-trip to themselves; NaNs are excluded
    np.testing.assert_array_equal(back, b[finite])


# ------------------------------------------------------------- expert FFN

def _rand_expert(H, I, seed, lo=118, hi=124):
    rng = np.random.default_rng(seed)
    codes = np.frombuffer(rng.bytes(3 * I * H // 2), dtype=np.uint8).copy()
    scales = rng.integers(lo, hi + 1, size=3 * I * H // 32, dtype=np.uint8)
    x = synth.f32_to_bf16_bits(rng.standard_normal(H, dtype=np.float32))
    return codes, scales, x


def _bruteforce_expert(x, codes, scales, H, I):
    mc, ms = I * H // 2, I * H // 32
    Wg = unpack_dense(codes[:mc], scales[:ms], I, H)
    Wu = unpack_dense(codes[mc:2 * mc], scales[ms:2 * ms], I, H)
    Wd = unpack_dense(codes[2 * mc:], scales[2 * ms:], H, I)
    xf = bf16_f64(x)
    g = bf16_f64(bf16_via_f32(Wg @ xf))
    u = bf16_f64(bf16_via_f32(Wu @ xf))
    s = bf16_f64(bf16_via_f32(g / (1.0 + np.exp(-g))))
    h = bf16_via_f32(s * u)
    o = bf16_via_f32(Wd @ bf16_f64(h))
    return h, o


@pytest.mark.parametrize("H,I,seed", [(64, 32, 0), (128, 96, 1), (512, 384, 2)])
def test_expert_matches_dense_bruteforce(H, I, seed):
    codes, scales, x = _rand_expert(H, I, seed)
    h, o = oracle.expert(x, codes, scales, H, I)
    hb, ob = _bruteforce_expert(x, codes, scales, H, I)
    # binary32 detours in the brute force may double-round a value sitting
    # within 2^-24 of a BF16 tie: allow one ulp on a handful of elements
    dh, do = ulp_diff(h, hb), ulp_diff(o, ob)
    assert dh.max() <= 1 and (dh > 0).sum() <= max(1, I // 500)
    assert do.max() <= 1 and (do > 0).sum() <= max(1, H // 500)
    # and the structure matters: gate/up swapped gives a different answer
    mc = I * H // 2
    ms = I * H // 32
    swapped = np.concatenate([codes[mc:2 * mc], codes[:mc], codes[2 * mc:]])
    sw_s = np.concatenate([scales[ms:2 * ms], scales[:ms], scales[2 * ms:]])
    h2, _ = oracle.expert(x, swapped, sw_s, H, I)
    assert (ulp_diff(h, h2) > 1).mean() > 0.5


def test_expert_zero_codes_give_zero():
    H, I = 64, 32
    codes, scales, x = _rand_expert(H, I, 3)
    h, o = oracle.expert(x, np.zeros_like(codes), scales, H, I)
    assert not np.any(h & 0x7FFF) and not np.any(o & 0x7FFF)


def test_expert_down_scale_doubling_doubles_output():
    H, I = 128, 64
    codes, scales, x = _rand_expert(H, I, 4)
    _, o = oracle.expert(x, codes, scales, H, I)
    s2 = scales.copy()
    s2[2 * I * H // 32:] += 1
    _, o2 = oracle.expert(x, codes, s2, H, I)
    np.testing.assert_array_equal(bf16_f64(o2), 2.0 * bf16_f64(o))


# ------------------------------------------------------------------ router

def test_route_matches_stable_sort_and_softmax():
    rng = np.random.default_rng(11)
    for E, k in ((16, 4), (64, 4), (8, 8), (32, 1)):
        H = 256
        x = synth.f32_to_bf16_bits(rng.standard_normal((6, H), dtype=np.float32))
        Wr = synth.f32_to_bf16_bits(rng.standard_normal((E, H), dtype=np.float32) * 0.02)
        ids, w, lg = oracle.route(x, Wr, None, k)
        ref_lg = bf16_f64(x) @ bf16_f64(Wr).T
        np.testing.assert_allclose(lg, ref_lg, rtol=1e-12, atol=1e-12)
        order = np.argsort(-lg, axis=1, kind="stable")[:, :k]
        np.testing.assert_array_equal(ids, order)
        ref_w = softmax(np.take_along_axis(lg, order, axis=1), axis=1)
        np.testing.assert_allclose(w, ref_w, rtol=1e-14, atol=1e-15)
        np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=1e-14)
        assert np.all(np.diff(w, axis=1) <= 0)


def test_route_ties_go_to_lower_id():
    lg = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, 2.0, -1.0, 0.0]])
    ids, w = oracle.select_topk(lg, 4)
    assert ids.tolist() == [[1, 3, 5, 2]]
    assert w[0, 0] == w[0, 1] == w[0, 2]


def test_route_bias_is_added_to_logits():
    rng = np.random.default_rng(12)
    E, H, k = 32, 128, 4
    x = synth.f32_to_bf16_bits(rng.standard_normal((3, H), dtype=np.float32))
    Wr = synth.f32_to_bf16_bits(rng.standard_normal((E, H), dtype=np.float32) * 0.02)
    b = rng.standard_normal(E).astype(np.float32)
    ids, w, lg = oracle.route(x, Wr, b, k)
    _, _, lg0 = oracle.route(x, Wr, None, k)
    np.testing.assert_allclose(lg, lg0 + b.astype(np.float64), rtol=0, atol=1e-12)
    # a huge bias on one expert forces it to slot 0
    b2 = np.zeros(E, dtype=np.float32)
    b2[17] = 1e3
    ids2, w2, _ = oracle.route(x, Wr, b2, k)
    assert np.all(ids2[:, 0] == 17) and np.all(w2[:, 0] > 0.999)


def test_sigmoid_route_hand_worked_example():
    """Logits whose sigmoids are exact small fractions: sigmoid(0) = 1/2,
    sigmoid(ln 3) = 3/4, sigmoid(ln 1/3) = 1/4, sigmoid(ln 9) = 9/10.
    Without bias the top-2 are experts 3 (0.9) and 1 (0.75), coefficients
    0.9/1.65 and 0.75/1.65.  A bias of +0.7 on expert 2 (key 0.95) and -0.5
    on expert 3 (key 0.4) selects experts 2 and 1 instead, and the
    coefficients still come from the unbiased scores: 0.25/1.0, 0.75/1.0."""
    lg = np.array([[0.0, np.log(3.0), np.log(1.0 / 3.0), np.log(9.0)]])
    ids, w = oracle.select_topk_sigmoid(lg, None, 2)
    assert ids.tolist() == [[3, 1]]
    np.testing.assert_allclose(w[0], [0.9 / 1.65, 0.75 / 1.65], rtol=1e-14)
    bias = np.array([0.0, 0.0, 0.7, -0.5], dtype=np.float32)
    ids, w = oracle.select_topk_sigmoid(lg, bias, 2)
    assert ids.tolist() == [[2, 1]]
    np.testing.assert_allclose(w[0], [0.25, 0.75], rtol=1e-14)
    # k = E: every expert, coefficients 0.5, 0.75, 0.25, 0.9 over 2.4
    ids, w = oracle.select_topk_sigmoid(lg, None, 4)
    assert ids.tolist() == [[3, 1, 0, 2]]
    np.testing.assert_allclose(w[0], np.array([0.9, 0.75, 0.5, 0.25]) / 2.4, rtol=1e-14)


def test_sigmoid_route_without_bias_selects_as_softmax_route():
    """The sigmoid is increasing: without bias both scorings select the same
    experts in the same order (their coefficients differ)."""
    rng = np.random.default_rng(13)
    lg = rng.standard_normal((50, 64)) * 3.0
    ids_s, w_s = oracle.select_topk_sigmoid(lg, None, 4)
    ids_m, _ = oracle.select_topk(lg, 4)
    np.testing.assert_array_equal(ids_s, ids_m)
    np.testing.assert_allclose(w_s.sum(axis=1), 1.0, rtol=1e-14)
    assert np.all(np.diff(w_s, axis=1) <= 0)


def test_sigmoid_route_ties_and_logits_unbiased():
    lg = np.array([[0.5, 2.0, 1.0, 2.0, 1.0, 2.0, -1.0, 0.0]])
    ids, w = oracle.select_topk_sigmoid(lg, None, 4)
    assert ids.tolist() == [[1, 3, 5, 2]]
    assert w[0, 0] == w[0, 1] == w[0, 2]
    rng = np.random.default_rng(14)
    E, H, k = 32, 128, 4
    x = synth.f32_to_bf16_bits(rng.standard_normal((3, H), dtype=np.float32))
    Wr = synth.f32_to_bf16_bits(rng.standard_normal((E, H), dtype=np.float32) * 0.02)
    b = rng.standard_normal(E).astype(np.float32)
    ids, w, lg = oracle.route(x, Wr, b, k, sigmoid=True)
    _, _, lg0 = oracle.route(x, Wr, None, k)
    np.testing.assert_array_equal(lg, lg0)  # the bias does not enter the logits
    ids2, w2 = oracle.select_topk_sigmoid(lg0, b, k)
    np.testing.assert_array_equal(ids, ids2)
    np.testing.assert_array_equal(w, w2)
    # a large bias on one expert forces it into slot 0 whatever its score
    b2 = np.zeros(E, dtype=np.float32)
    b2[17] = 10.0
    ids3, w3, _ = oracle.route(x, Wr, b2, k, sigmoid=True)
    assert np.all(ids3[:, 0] == 17)
    s = 1.0 / (1.0 + np.exp(-lg0))
    np.testing.assert_allclose(w3[:, 0], s[:, 17] / np.take_along_axis(s, ids3, 1).sum(1),
                               rtol=1e-13)


# ----------------------------------------------------------------- combine

def test_combine_hand_derived_examples(golden):
    for row in golden("combine_sequential.txt"):
        name, o_s, w_s, r_s, y_s = [s.strip() for s in row.split("|")]
        o = np.array([int(v, 16) for v in o_s.split()], dtype=np.uint16)
        w = np.array([float(v) for v in w_s.split()])
        H = 1
        r = None if r_s == "-" else np.array([int(r_s, 16)], dtype=np.uint16)
        y = oracle.combine(o.reshape(-1, H), w, residual=r)
        assert int(y[0]) == int(y_s, 16), name


def test_combine_single_slot_weight_one_is_identity():
    rng = np.random.default_rng(5)
    o = synth.f32_to_bf16_bits(rng.standard_normal((4, 300), dtype=np.float32))
    y = oracle.combine(o, np.array([1.0, 0.0, 0.0, 0.0]))
    np.testing.assert_array_equal(bf16_f64(y), bf16_f64(o[0]) + 0.0)


# ------------------------------------------------------------------- layer

def test_moe_layer_is_route_then_forward():
    sh = synth.LayerShape(E=8, H=128, I=64, top_k=4)
    L = synth.make_layer(sh, seed=3)
    x = synth.make_tokens(3, sh.H, seed=3)
    ids, w, y = oracle.moe_layer(x, L.router_w, None, L.codes, L.scales,
                                 sh.E, sh.H, sh.I, sh.top_k)
    ids2, w2, _ = oracle.route(x, L.router_w, None, sh.top_k)
    np.testing.assert_array_equal(ids, ids2)
    y2, o = oracle.moe_forward(x, ids2, w2, L.codes, L.scales, sh.E, sh.H, sh.I,
                               want_o=True)
    np.testing.assert_array_equal(y, y2)
    # each slot's o is the single-expert oracle on that expert
    for t in range(3):
        for j in range(4):
            e = ids[t, j]
            _, oe = oracle.expert(x[t], L.codes[e], L.scales[e], sh.H, sh.I)
            np.testing.assert_array_equal(o[t, j], oe)
    # weight one on slot 0 reduces the layer to that expert
    w1 = np.zeros_like(w2)
    w1[:, 0] = 1.0
    y1 = oracle.moe_forward(x, ids2, w1, L.codes, L.scales, sh.E, sh.H, sh.I)
    np.testing.assert_array_equal(bf16_f64(y1), bf16_f64(o[:, 0]) + 0.0)


def test_invalid_id_slot_contributes_zero():
    sh = synth.LayerShape(E=8, H=64, I=32, top_k=2)
    L = synth.make_layer(sh, seed=4)
    x = synth.make_tokens(1, sh.H, seed=4)
    w = np.array([[0.7, 0.3]])
    y_bad, o = oracle.moe_forward(x, np.array([[2, 99]]), w, L.codes, L.scales,
                                  sh.E, sh.H, sh.I, want_o=True)
    assert not np.any(o[0, 1] & 0x7FFF)
    y_one = oracle.moe_forward(x, np.array([[2, 99]]), np.array([[0.7, 0.0]]),
                               L.codes, L.scales, sh.E, sh.H, sh.I)
    np.testing.assert_array_equal(y_bad, y_one)


# ------------------------------------------------------------------- stack

def test_rmsnorm_closed_forms():
    H = 2048
    one = np.full((1, H), 0x3F80, dtype=np.uint16)             # all 1.0
    xn = oracle.rmsnorm(one)
    assert np.all(xn == 0x3F80)       # 1/sqrt(1+1e-6) rounds to 1.0
    r = np.zeros((1, H), dtype=np.uint16)
    r[0, 0] = 0x4040                  # 3.0, rest 0 -> mean(r^2) = 9/H
    xn = oracle.rmsnorm(r)
    exp = 3.0 / math.sqrt(9.0 / H + 1e-6)
    assert bf16_f64(xn[0, 0]) == bf16_f64(bf16_via_f32(np.array([exp])))[0]
    assert np.all(xn[0, 1:] == 0)


def test_stack_one_layer_is_norm_layer_residual():
    sh = synth.LayerShape(E=8, H=128, I=64, top_k=4)
    L = synth.make_layer(sh, seed=6)
    r = synth.make_tokens(2, sh.H, seed=6)
    r_out, ids = oracle.stack_step(r, [L])
    xn = oracle.rmsnorm(r)
    ids2, w2, y = oracle.moe_layer(xn, L.router_w, None, L.codes, L.scales,
                                   sh.E, sh.H, sh.I, sh.top_k)
    np.testing.assert_array_equal(ids[0], ids2)
    y_plain = oracle.moe_forward(xn, ids2, w2, L.codes, L.scales, sh.E, sh.H, sh.I)
    want = oracle.bf16_from_f64_array(bf16_f64(r) + bf16_f64(y_plain))
    np.testing.assert_array_equal(r_out, want)


# ------------------------------------------------------------ closed forms

def test_closed_forms(golden):
    g = dict(row.split() for row in golden("closed_forms.txt"))
    h, mi, ex, k, nl = (int(g[n]) for n in ("hidden", "moe_inter", "experts", "top_k", "moe_layers"))
    per_expert = 3 * h * mi
    assert per_expert == int(g["per_expert_params"])
    all_e = per_expert * ex * nl
    active = per_expert * k * nl
    always_on = int(g["total_params"]) - all_e
    assert round(all_e / 1e9, 2) == float(g["all_expert_params_rounded_billions"])
    assert round(active / 1e9, 2) == float(g["active_expert_params_rounded_billions"])
    assert round(always_on / 1e9, 2) == float(g["always_on_params_rounded_billions"])
    assert round((always_on + active) / 1e9, 4) == float(g["active_total_rounded_4dp_billions"])
    # storage of the shapes used everywhere in this repository
    sh = synth.L24B
    assert (sh.H, sh.I, sh.E, sh.top_k) == (h, mi, ex, k)
    assert 3 * sh.I * sh.H == per_expert
    packed = sh.codes_per_expert + sh.scales_per_expert
    assert packed == int(g["packed_bytes_per_expert"])
    assert packed * 2 == per_expert + per_expert // 16      # 0.5 + 1/32 B/weight
    assert k * packed == int(g["streamed_bytes_per_token_layer"])
    # the oracle consumes exactly one expert's bytes per selected slot
    codes, scales = synth.make_expert_weights(synth.LayerShape(E=1, H=64, I=32), np.random.default_rng(0))
    assert codes.size == 3 * 64 * 32 // 2 and scales.size == 3 * 64 * 32 // 32


# --------------------------------------------------------------- NVFP4

def e4m3_torch(b):
    """FP8 E4M3 bytes decoded by torch's own float8_e4m3fn dtype."""
    t = torch.from_numpy(np.asarray(b, dtype=np.uint8).copy()).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def unpack_dense_nvfp4(codes_m, scales_m, g, rows, K):
    """Independent unpacker: packed [rows][K/2] + E4M3 [rows][K/16] (decoded
    by torch) times the global multiplier g -> f64."""
    b = np.asarray(codes_m, dtype=np.uint8).reshape(rows, K // 2)
    nib = np.empty((rows, K), dtype=np.int64)
    nib[:, 0::2] = b & 0x0F
    nib[:, 1::2] = b >> 4
    table = np.array([e2m1_bitfield(c) for c in range(16)])
    sc = np.repeat(e4m3_torch(scales_m).reshape(rows, K // 16), 16, axis=1)
    return table[nib] * sc * float(np.float32(g))


def test_e4m3_matches_torch_float8_all_bytes():
    b = np.arange(256, dtype=np.uint8)
    want = e4m3_torch(b)
    got = np.array([oracle.e4m3_value(int(v)) for v in b])
    nan = np.isnan(want)
    assert nan.sum() == 2 and np.array_equal(np.isnan(got), nan)  # 0x7F, 0xFF
    np.testing.assert_array_equal(got[~nan], want[~nan])
    assert np.signbit(got[0x80]) and got[0x80] == 0.0
    # closed forms: 1.0, the largest finite 448, the smallest subnormal 2^-9
    assert (got[0x38], got[0x7E], got[0x01]) == (1.0, 448.0, 2.0 ** -9)


def test_dequant_nvfp4_block_indexing():
    """Code 2 (value 1.0) everywhere, a different E4M3 scale per 16-element
    block: element j is scale[j // 16] times the multiplier."""
    n = 64
    codes = np.full(n // 2, 0x22, dtype=np.uint8)
    scales = np.array([0x38, 0x40, 0x30, 0xB8], dtype=np.uint8)  # 1, 2, 0.5, -1
    out = oracle.dequant_nvfp4(codes, scales, 0.75, n)
    np.testing.assert_array_equal(out, np.repeat([0.75, 1.5, 0.375, -0.75], 16))


def _rand_expert_nvfp4(H, I, seed):
    rng = synth.rng_for(seed, 99)
    shape = synth.LayerShape(E=1, H=H, I=I)
    codes, scales, gs = synth.make_expert_weights_nvfp4(shape, rng)
    x = synth.f32_to_bf16_bits(rng.standard_normal(H, dtype=np.float32))
    return codes[0], scales[0], gs[0], x


@pytest.mark.parametrize("H,I,seed", [(64, 32, 0), (128, 96, 1), (512, 384, 2)])
def test_expert_nvfp4_matches_dense_bruteforce(H, I, seed):
    codes, scales, gs, x = _rand_expert_nvfp4(H, I, seed)
    h, o = oracle.expert_nvfp4(x, codes, scales, gs, H, I)
    mc, ms = I * H // 2, I * H // 16
    Wg = unpack_dense_nvfp4(codes[:mc], scales[:ms], gs[0], I, H)
    Wu = unpack_dense_nvfp4(codes[mc:2 * mc], scales[ms:2 * ms], gs[0], I, H)
    Wd = unpack_dense_nvfp4(codes[2 * mc:], scales[2 * ms:], gs[1], H, I)
    xf = bf16_f64(x)
    g = bf16_f64(bf16_via_f32(Wg @ xf))
    u = bf16_f64(bf16_via_f32(Wu @ xf))
    s = bf16_f64(bf16_via_f32(g / (1.0 + np.exp(-g))))
    hb = bf16_via_f32(s * u)
    ob = bf16_via_f32(Wd @ bf16_f64(hb))
    dh, do = ulp_diff(h, hb), ulp_diff(o, ob)
    assert dh.max() <= 1 and (dh > 0).sum() <= max(1, I // 500)
    assert do.max() <= 1 and (do > 0).sum() <= max(1, H // 500)
    # the gate/up multiplier is shared, the down one separate: swapping them
    # changes the answer
    h2, o2 = oracle.expert_nvfp4(x, codes, scales, gs[::-1].copy(), H, I)
    assert (ulp_diff(o, o2) > 1).mean() > 0.3


def test_expert_nvfp4_down_multiplier_doubling_doubles_output():
    H, I = 128, 64
    codes, scales, gs, x = _rand_expert_nvfp4(H, I, 4)
    _, o = oracle.expert_nvfp4(x, codes, scales, gs, H, I)
    gs2 = gs.copy()
    gs2[1] *= 2
    _, o2 = oracle.expert_nvfp4(x, codes, scales, gs2, H, I)
    np.testing.assert_array_equal(bf16_f64(o2), 2.0 * bf16_f64(o))


def test_nvfp4_reduces_to_mxfp4_when_scales_coincide():
    """Block scales equal to the power of two of an E8M0 group scale (both
    16-blocks of the group) and unit multipliers give the MXFP4 layer."""
    shape = synth.LayerShape(E=4, H=128, I=96)
    L = synth.make_layer(shape, seed=5)
    # E8M0 118..124 = 2^-9 .. 2^-3: E4M3 0x01, 0x02, 0x04 (subnormal), then
    # 0x08, 0x10, 0x18, 0x20
    e4m3_of = {118: 0x01, 119: 0x02, 120: 0x04, 121: 0x08, 122: 0x10, 123: 0x18, 124: 0x20}
    nv_scales = np.vectorize(e4m3_of.get)(np.repeat(L.scales, 2, axis=1)).astype(np.uint8)
    gs = np.ones((shape.E, 2), dtype=np.float32)
    x = synth.make_tokens(3, shape.H, seed=5)
    ids = np.array([[0, 1, 2, 3], [3, 1, 0, 2], [2, 2, 1, 0]], dtype=np.int32)
    w = np.array([[0.4, 0.3, 0.2, 0.1]] * 3)
    y_mx = oracle.moe_forward(x, ids, w, L.codes, L.scales, shape.E, shape.H, shape.I)
    y_nv = oracle.moe_forward_nvfp4(x, ids, w, L.codes, nv_scales, gs, shape.E, shape.H,
                                    shape.I)
    np.testing.assert_array_equal(y_nv, y_mx)


# ---------------------------------------------------------------- sym8

def unpack_dense_sym8(q_m, scales_m, rows, K):
    """Independent unpacker: int8 [rows][K] times the binary16 scale of each
    32-element block, decoded by numpy's own float16 -> f64."""
    q = np.asarray(q_m).view(np.int8).reshape(rows, K).astype(np.float64)
    s = np.asarray(scales_m, dtype=np.uint16).view(np.float16).astype(np.float64)
    return q * np.repeat(s.reshape(rows, K // 32), 32, axis=1)


def test_f16_matches_numpy_binary16_all_patterns():
    b = np.arange(65536, dtype=np.uint32)
    want = b.astype(np.uint16).view(np.float16).astype(np.float64)
    got = np.array([oracle.f16_value(int(v)) for v in b])
    nan = np.isnan(want)
    assert nan.sum() == 2 * 1023 and np.array_equal(np.isnan(got), nan)
    np.testing.assert_array_equal(got[~nan], want[~nan])
    # closed forms: 1.0, the largest finite 65504, the least subnormal 2^-24,
    # the least normal 2^-14, infinities, a signed zero
    assert (got[0x3C00], got[0x7BFF], got[0x0001], got[0x0400]) == (1.0, 65504.0, 2.0 ** -24,
                                                                    2.0 ** -14)
    assert got[0x7C00] == np.inf and got[0xFC00] == -np.inf
    assert np.signbit(got[0x8000]) and got[0x8000] == 0.0


def test_dequant_sym8_block_indexing_and_sign():
    """q = j - 64 over 128 elements (every sign, -128 included), a different
    binary16 scale per 32-element block: element j is (j - 64) times
    scale[j // 32]."""
    n = 128
    q = (np.arange(n) - 64).astype(np.int8)
    scales = np.array([0x3C00, 0x4000, 0x3800, 0xBC00], dtype=np.uint16)  # 1, 2, 0.5, -1
    out = oracle.dequant_sym8(q, scales, n)
    want = (np.arange(n) - 64) * np.repeat([1.0, 2.0, 0.5, -1.0], 32)
    np.testing.assert_array_equal(out, want)
    assert out[0] == -64.0 and out[127] == -63.0


def _rand_expert_sym8(H, I, seed):
    rng = synth.rng_for(seed, 98)
    shape = synth.LayerShape(E=1, H=H, I=I)
    q, scales = synth.make_expert_weights_sym8(shape, rng)
    x = synth.f32_to_bf16_bits(rng.standard_normal(H, dtype=np.float32))
    return q[0], scales[0], x


@pytest.mark.parametrize("H,I,seed", [(64, 32, 0), (128, 96, 1), (512, 384, 2)])
def test_expert_sym8_matches_dense_bruteforce(H, I, seed):
    q, scales, x = _rand_expert_sym8(H, I, seed)
    h, o = oracle.expert_sym8(x, q, scales, H, I)
    mc, ms = I * H, I * H // 32
    Wg = unpack_dense_sym8(q[:mc], scales[:ms], I, H)
    Wu = unpack_dense_sym8(q[mc:2 * mc], scales[ms:2 * ms], I, H)
    Wd = unpack_dense_sym8(q[2 * mc:], scales[2 * ms:], H, I)
    xf = bf16_f64(x)
    g = bf16_f64(bf16_via_f32(Wg @ xf))
    u = bf16_f64(bf16_via_f32(Wu @ xf))
    s = bf16_f64(bf16_via_f32(g / (1.0 + np.exp(-g))))
    hb = bf16_via_f32(s * u)
    ob = bf16_via_f32(Wd @ bf16_f64(hb))
    dh, do = ulp_diff(h, hb), ulp_diff(o, ob)
    assert dh.max() <= 1 and (dh > 0).sum() <= max(1, I // 500)
    assert do.max() <= 1 and (do > 0).sum() <= max(1, H // 500)
    # the structure matters: gate/up swapped gives a different answer
    q_sw = np.concatenate([q[mc:2 * mc], q[:mc], q[2 * mc:]])
    s_sw = np.concatenate([scales[ms:2 * ms], scales[:ms], scales[2 * ms:]])
    h2, _ = oracle.expert_sym8(x, q_sw, s_sw, H, I)
    assert (ulp_diff(h, h2) > 1).mean() > 0.5


def test_expert_sym8_negated_down_weights_negate_output():
    """q of the down matrix negated (the grid is symmetric): o changes sign
    exactly, h does not change."""
    H, I = 128, 64
    q, scales, x = _rand_expert_sym8(H, I, 5)
    h, o = oracle.expert_sym8(x, q, scales, H, I)
    q2 = q.copy()
    q2[2 * I * H:] = -q2[2 * I * H:]
    h2, o2 = oracle.expert_sym8(x, q2, scales, H, I)
    np.testing.assert_array_equal(h2, h)
    np.testing.assert_array_equal(bf16_f64(o2), -bf16_f64(o))


def test_sym8_reduces_to_mxfp4_when_values_coincide():
    """Each E2M1 code c with E8M0 group exponent e is the int8 value 2 e2m1(c)
    with the binary16 scale 2^(e - 128): the sym8 layer then equals the MXFP4
    layer bit for bit (same weights, same summation order)."""
    shape = synth.LayerShape(E=4, H=128, I=96)
    L = synth.make_layer(shape, seed=6)
    n = 3 * shape.I * shape.H
    nib = np.empty((shape.E, n), dtype=np.int64)
    nib[:, 0::2] = L.codes & 0x0F
    nib[:, 1::2] = L.codes >> 4
    twice = np.array([2 * e2m1_bitfield(c) for c in range(16)])
    q = twice[nib].astype(np.int8)
    # 2^(e - 128) for e = 118 .. 124 is a normal binary16 (exponent field e - 113)
    f16 = ((L.scales.astype(np.uint16) - 113) << 10).astype(np.uint16)
    assert np.array_equal(f16.view(np.float16).astype(np.float64),
                          2.0 ** (L.scales.astype(np.float64) - 128))
    x = synth.make_tokens(3, shape.H, seed=6)
    ids = np.array([[0, 1, 2, 3], [3, 1, 0, 2], [2, 9, 1, 0]], dtype=np.int32)  # 9: invalid
    w = np.array([[0.4, 0.3, 0.2, 0.1]] * 3)
    r = synth.make_tokens(3, shape.H, seed=7)
    y_mx, o_mx, h_mx = oracle.moe_forward(x, ids, w, L.codes, L.scales, shape.E, shape.H,
                                          shape.I, residual=r, want_o=True, want_h=True)
    y_s8, o_s8, h_s8 = oracle.moe_forward_sym8(x, ids, w, q, f16, shape.E, shape.H, shape.I,
                                               residual=r, want_o=True, want_h=True)
    np.testing.assert_array_equal(h_s8, h_mx)
    np.testing.assert_array_equal(o_s8, o_mx)
    np.testing.assert_array_equal(y_s8, y_mx)
