"""Pins of the oracle's FP8 (e4m3) expert path.

The e4m3 value of every code and the rounding of fp32 values are checked
against the library's float8_e4m3fn type and against a nearest-value search
over the whole code table (oracle/loop_over_experts.py); the row quantizer
against the closed facts of its definition (the row's largest magnitude maps
to 448, every element within half an e4m3 step, zero rows stay zero); the FP8
layer against the independent loop-over-experts formulation.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import loop_over_experts as loe


def _codes_of(a):
    """e4m3 codes of float32 values through the library cast."""
    return torch.from_numpy(np.ascontiguousarray(a, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_value_of_every_code_matches_library():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_value(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    assert np.array_equal(np.isnan(ours), np.isnan(lib))
    ok = ~np.isnan(lib)
    assert np.array_equal(ours[ok], lib[ok])
    # the format's landmarks: largest finite 448, smallest subnormal 2^-9,
    # smallest normal 2^-6, one, and the two NaN codes
    assert ours[0x7E] == 448.0 and ours[0x01] == 2.0 ** -9 and ours[0x08] == 2.0 ** -6
    assert ours[0x38] == 1.0 and ours[0xB8] == -1.0
    assert np.isnan(ours[0x7F]) and np.isnan(ours[0xFF])


def _rounding_probe():
    rng = np.random.default_rng(3)
    vals = [rng.standard_normal(4000) * s for s in (1e-4, 1e-2, 1.0, 30.0, 300.0)]
    mags = loe.E4M3[:127]
    mids = (mags[:-1] + mags[1:]) / 2.0           # exact ties between neighbours
    vals += [mids, -mids, mags, -mags, mids * (1 + 2.0 ** -20), mids * (1 - 2.0 ** -20)]
    vals.append(np.array([0.0, -0.0, 447.0, 448.0, 449.0, 463.9, 464.0, 1e6, -1e6, 2.0 ** -10, 2.0 ** -11,
                          -2.0 ** -12, 3 * 2.0 ** -11]))
    return np.concatenate(vals).astype(np.float32)


def test_e4m3_round_matches_nearest_search():
    q = _rounding_probe()
    assert np.array_equal(oracle.e4m3_round(q), loe.e4m3_nearest(q))


def test_e4m3_round_matches_library_cast():
    q = _rounding_probe()
    q = q[np.abs(q) <= 448.0]                      # the library's cast does not saturate
    assert np.array_equal(oracle.e4m3_round(q), _codes_of(q))


def test_e4m3_round_ties_go_to_even_and_saturate():
    mags = loe.E4M3[:127]
    mids = ((mags[:-1] + mags[1:]) / 2.0).astype(np.float32)
    codes = oracle.e4m3_round(mids)
    assert np.all(codes % 2 == 0)
    assert np.all(oracle.e4m3_round(np.array([449.0, 1e30, -1e30], np.float32)) == [0x7E, 0x7E, 0xFE])
    # sign kept on values that round to zero
    assert list(oracle.e4m3_round(np.array([-1e-9, 1e-9, -0.0], np.float32))) == [0x80, 0x00, 0x80]


def test_quantize_rows_closed_facts():
    rng = np.random.default_rng(4)
    v = np.concatenate([rng.standard_normal((6, 70)) * s for s in (1e-3, 1.0, 1e3)]).astype(np.float32)
    v[2, :] = 0.0                                   # a zero row
    v[5, 10] = -50.0                                # a negative maximum
    codes, scale = oracle.quantize_rows(v)
    val = oracle.e4m3_value(codes)
    for r in range(v.shape[0]):
        amax = np.abs(v[r]).max()
        if amax == 0:
            assert scale[r] == 0 and not codes[r].any()
            continue
        assert np.abs(val[r]).max() == 448.0
        assert scale[r] == np.float32(amax) / np.float32(448.0)
        # every element within half a step of its binade (2^-4 relative), or
        # half the subnormal step below 2^-6
        q = v[r].astype(np.float64) * np.float64(np.float32(448.0) / np.float32(amax))
        err = np.abs(val[r] - q)
        assert np.all(err <= np.maximum(np.abs(q) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-12))
    # the independent formulation gives the same bytes
    c2, s2 = loe.quantize_rows_np(v)
    assert np.array_equal(codes, c2) and np.array_equal(scale, s2)


def fp8_case(rng, T, d, E, F, *, act, shared=0):
    """Random bf16 x, fp32 router, and FP8 experts (codes of N(0,1) draws
    through the library cast, per-channel scales around 1/sqrt(fan_in))."""
    x32 = rng.standard_normal((T, d)).astype(np.float32)
    x = (x32.view(np.uint32) >> 16).astype(np.uint16)
    Wr = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)

    def mat(rows_shape, fan_in, name, w):
        w[name] = _codes_of(rng.standard_normal(rows_shape + (fan_in,)))
        w[name + "_scale"] = (rng.uniform(0.5, 1.5, rows_shape) / np.sqrt(fan_in)).astype(np.float32)

    w = {}
    mat((E, F), d, "W1", w)
    mat((E, d), F, "W2", w)
    if act == "swiglu":
        mat((E, F), d, "Wu", w)
    else:
        w["b1"] = rng.uniform(-0.01, 0.01, (E, F)).astype(np.float32)
        w["b2"] = rng.uniform(-0.01, 0.01, (E, d)).astype(np.float32)
    if shared:
        mat((shared,), d, "Wsg", w)
        mat((d,), shared, "Wsd", w)
        if act == "swiglu":
            mat((shared,), d, "Wsu", w)
    return x, Wr, w


FP8_CASES = [
    dict(act="gelu", score="softmax", renorm=1, k=2, E=6, cap=-1.0, shared=0),
    dict(act="swiglu", score="softmax", renorm=1, k=3, E=8, cap=0.7, shared=0),
    dict(act="swiglu", score="sigmoid", renorm=1, k=4, E=12, cap=-1.0, shared=40),
]


@pytest.mark.parametrize("case", FP8_CASES, ids=lambda c: "%s-k%d-cap%s-sh%d" % (
    c["act"], c["k"], c["cap"], c["shared"]))
def test_fp8_layer_agrees_with_loop_over_experts(case):
    rng = np.random.default_rng(case["E"] * 7 + case["k"])
    T, d, F = 40, 48, 56
    E, k = case["E"], case["k"]
    x, Wr, w = fp8_case(rng, T, d, E, F, act=case["act"], shared=case["shared"])
    sb = rng.normal(0, 0.1, E).astype(np.float32) if case["score"] == "sigmoid" else None
    C = oracle.capacity(case["cap"], k, T, E)
    dims = oracle.make_dims(T, d, E, F, k, x_dtype="bf16", act=case["act"], score=case["score"],
                            renorm=case["renorm"], capacity=C, d_ff_shared=case["shared"])
    r = oracle.route(dims, x, Wr, None, sb)
    dp = oracle.dispatch(dims, r["idx"])
    x8, xs = oracle.quantize_rows(oracle.bf16_bits_to_f64(x).astype(np.float32))
    y = oracle.layer_tokens_fp8(dims, x8, xs, w, r["idx"], r["gate"], dp["row_of"], np.arange(T))
    ref = loe.layer_fp8(x, Wr, w, k, act=case["act"], score=case["score"], renorm=case["renorm"],
                        capacity=C, sel_bias=sb)
    assert np.array_equal(x8, ref["x8"]) and np.array_equal(xs, ref["xs"])
    np.testing.assert_array_equal(r["idx"], ref["idx"])
    np.testing.assert_allclose(y, ref["y"], rtol=1e-10, atol=1e-12)


def test_fp8_expert_scales_enter_linearly():
    """Doubling the down projection's channel scales doubles the output
    exactly; so does doubling SwiGLU's up-projection scales (H = SiLU(g) * u
    doubles exactly, its bf16 rounding and row quantization keep the same
    codes with twice the scale)."""
    rng = np.random.default_rng(9)
    T, d, E, F = 6, 32, 2, 40
    x, Wr, w = fp8_case(rng, T, d, E, F, act="swiglu")
    dims = oracle.make_dims(T, d, E, F, 1, x_dtype="bf16", act="swiglu")
    x8, xs = oracle.quantize_rows(oracle.bf16_bits_to_f64(x).astype(np.float32))
    tok = np.arange(T, dtype=np.int32)
    ex = np.zeros(T, np.int32)
    base = oracle.expert_apply_fp8(dims, x8, xs, w, tok, ex)
    w2 = dict(w)
    w2["W2_scale"] = w["W2_scale"] * np.float32(2)
    assert np.array_equal(oracle.expert_apply_fp8(dims, x8, xs, w2, tok, ex), 2 * base)
    w3 = dict(w)
    w3["Wu_scale"] = w["Wu_scale"] * np.float32(2)
    assert np.array_equal(oracle.expert_apply_fp8(dims, x8, xs, w3, tok, ex), 2 * base)
