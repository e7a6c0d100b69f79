"""Pins of the oracle's block-scaled (MX) FP8 expert path.

The MX quantizer against the closed facts of its definition (each block's
largest magnitude lands in [256, 512) times the block scale, the scale is a
power of two in [2^-127, 2^127], every element within half an e4m3 step of its
scaled value unless it saturates at 448, zero blocks stay zero) and against an
independent formulation that finds each block's exponent by comparing with
every power of two and each code by a search over the e4m3 table; the MX layer
against the loop-over-experts formulation on dequantized matrices; the scales
entering as exact powers of two.
"""
import numpy as np
import pytest

import oracle
from oracle import loop_over_experts as loe

from test_oracle_fp8_pins import _codes_of


def _probe_blocks(rng):
    v = [rng.standard_normal((6, 96)) * s for s in (1e-30, 1e-3, 1.0, 1e3, 1e30)]
    v = np.concatenate(v).astype(np.float32)
    v[3, 32:64] = 0.0                                       # a zero block
    v[4, 0:32] = np.float32(448.0) * rng.uniform(-1, 1, 32).astype(np.float32)
    v[4, 5] = np.float32(448.0)                             # amax exactly 448: X = 0
    v[5, 64:96] = np.float32(2.0 ** -130)                   # subnormal block: X clamps to -127
    v[7, 0:32] = np.float32(3.0e38)                         # near fp32's top: X = 119
    return v


def test_quantize_mx_closed_facts():
    v = _probe_blocks(np.random.default_rng(11))
    codes, scales = oracle.quantize_mx(v)
    assert codes.shape == v.shape and scales.shape == (v.shape[0], v.shape[1] // 32)
    val = oracle.e4m3_value(codes.ravel()).reshape(codes.shape)
    for r in range(v.shape[0]):
        for b in range(v.shape[1] // 32):
            blk = v[r, b * 32:(b + 1) * 32].astype(np.float64)
            cb = val[r, b * 32:(b + 1) * 32]
            X = int(scales[r, b]) - 127
            amax = np.abs(blk).max()
            if amax == 0:
                assert scales[r, b] == 0 and not codes[r, b * 32:(b + 1) * 32].any()
                continue
            q = blk / 2.0 ** X                              # exact
            if -127 < X:
                assert 256.0 <= np.abs(q).max() < 512.0, (r, b)
            # nearest code or saturation at 448; within half a step otherwise
            sat = np.abs(q) > 448.0
            assert np.all(np.abs(cb[sat]) == 448.0)
            err = np.abs(cb[~sat] - q[~sat])
            assert np.all(err <= np.maximum(np.abs(q[~sat]) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-12)), (r, b)
            assert np.all(np.signbit(cb[q != 0]) == np.signbit(q[q != 0]))
    assert scales[4, 0] == 127                              # amax = 448 -> 2^0
    assert scales[5, 2] == 0                                # clamped at 2^-127
    assert scales[7, 0] == 127 + 119                        # floor(log2 3e38) = 127 -> X = 119


def test_quantize_mx_matches_independent_search():
    v = _probe_blocks(np.random.default_rng(12))
    # exact ties between neighbouring codes after scaling by 2^-X = 2^-(-8): mids * 2^-8
    mags = loe.E4M3[:127]
    mids = ((mags[:-1] + mags[1:]) / 2.0)[:96] * 2.0 ** -8
    v[8, :] = mids.astype(np.float32)
    v[8, 31] = np.float32(448.0 * 2.0 ** -8)                # fixes X = -8 for the first block
    c1, s1 = oracle.quantize_mx(v)
    c2, s2 = loe.quantize_mx_np(v)
    assert np.array_equal(s1, s2)
    assert np.array_equal(c1, c2)


def test_quantize_mx_rejects_ragged_rows():
    with pytest.raises(ValueError):
        oracle.quantize_mx(np.ones((2, 40), np.float32))


def mx_case(rng, T, d, E, F, *, act, shared=0):
    """Random bf16 x, fp32 router, MX experts: e4m3 codes of N(0,1) draws with
    one random scale byte per 32 inputs around 1/sqrt(fan_in)."""
    x32 = rng.standard_normal((T, d)).astype(np.float32)
    x = (x32.view(np.uint32) >> 16).astype(np.uint16)
    Wr = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)
    w = {}

    def mat(rows_shape, fan_in, name):
        w[name] = _codes_of(rng.standard_normal(rows_shape + (fan_in,)))
        base = 127 - int(np.ceil(np.log2(np.sqrt(fan_in))))
        w[name + "_scale"] = rng.integers(base - 1, base + 2, rows_shape + (fan_in // 32,)).astype(np.uint8)

    mat((E, F), d, "W1")
    mat((E, d), F, "W2")
    if act == "swiglu":
        mat((E, F), d, "Wu")
    else:
        w["b1"] = rng.uniform(-0.01, 0.01, (E, F)).astype(np.float32)
        w["b2"] = rng.uniform(-0.01, 0.01, (E, d)).astype(np.float32)
    if shared:
        mat((shared,), d, "Wsg")
        mat((d,), shared, "Wsd")
        if act == "swiglu":
            mat((shared,), d, "Wsu")
    return x, Wr, w


MX_CASES = [
    dict(act="gelu", score="softmax", renorm=1, k=2, E=6, cap=-1.0, shared=0),
    dict(act="swiglu", score="softmax", renorm=1, k=3, E=8, cap=0.7, shared=0),
    dict(act="swiglu", score="sigmoid", renorm=1, k=4, E=12, cap=-1.0, shared=64),
]


@pytest.mark.parametrize("case", MX_CASES, ids=lambda c: "%s-k%d-cap%s-sh%d" % (
    c["act"], c["k"], c["cap"], c["shared"]))
def test_mx_layer_agrees_with_loop_over_experts(case):
    rng = np.random.default_rng(case["E"] * 5 + case["k"])
    T, d, F = 40, 64, 96
    E, k = case["E"], case["k"]
    x, Wr, w = mx_case(rng, T, d, E, F, act=case["act"], shared=case["shared"])
    sb = rng.normal(0, 0.1, E).astype(np.float32) if case["score"] == "sigmoid" else None
    C = oracle.capacity(case["cap"], k, T, E)
    dims = oracle.make_dims(T, d, E, F, k, x_dtype="bf16", act=case["act"], score=case["score"],
                            renorm=case["renorm"], capacity=C, d_ff_shared=case["shared"])
    r = oracle.route(dims, x, Wr, None, sb)
    dp = oracle.dispatch(dims, r["idx"])
    x8, xs = oracle.quantize_mx(oracle.bf16_bits_to_f64(x).astype(np.float32))
    y = oracle.layer_tokens_mx(dims, x8, xs, w, r["idx"], r["gate"], dp["row_of"], np.arange(T))
    ref = loe.layer_mx(x, Wr, w, k, act=case["act"], score=case["score"], renorm=case["renorm"],
                       capacity=C, sel_bias=sb)
    assert np.array_equal(x8, ref["x8"]) and np.array_equal(xs, ref["xs"])
    np.testing.assert_array_equal(r["idx"], ref["idx"])
    np.testing.assert_allclose(y, ref["y"], rtol=1e-10, atol=1e-12)


def test_mx_scales_enter_as_powers_of_two():
    """One more in every scale byte of the down projection doubles the output
    exactly; one more in every up-projection scale byte (SwiGLU) doubles H
    exactly, so its bf16 rounding and MX codes keep with the block scales one
    higher, and the output doubles exactly too."""
    rng = np.random.default_rng(13)
    T, d, E, F = 6, 64, 2, 64
    x, Wr, w = mx_case(rng, T, d, E, F, act="swiglu")
    dims = oracle.make_dims(T, d, E, F, 1, x_dtype="bf16", act="swiglu")
    x8, xs = oracle.quantize_mx(oracle.bf16_bits_to_f64(x).astype(np.float32))
    tok = np.arange(T, dtype=np.int32)
    ex = np.zeros(T, np.int32)
    base = oracle.expert_apply_mx(dims, x8, xs, w, tok, ex)
    w2 = dict(w, W2_scale=(w["W2_scale"] + 1).astype(np.uint8))
    np.testing.assert_array_equal(oracle.expert_apply_mx(dims, x8, xs, w2, tok, ex), 2.0 * base)
    wu = dict(w, Wu_scale=(w["Wu_scale"] + 1).astype(np.uint8))
    np.testing.assert_array_equal(oracle.expert_apply_mx(dims, x8, xs, wu, tok, ex), 2.0 * base)
