"""Pins of the oracle's INT4 weight-only expert path.

The weight decoding against closed facts (every nibble q + 8 with a unit scale
decodes to q exactly, power-of-two scales exactly, the low nibble is the even
input, one scale per 128 inputs, other scales rounded to the nearest bf16 of
q * s) and against an independent numpy decoding; the INT4 layer against the
loop-over-experts layer on the dequantized matrices; doubling the scales
doubling the output exactly.
"""
import numpy as np
import pytest

import oracle
from oracle import loop_over_experts as loe


def bf16_bits(v):
    return (np.asarray(v, np.float32).view(np.uint32) >> 16).astype(np.uint16)


def test_w4_decoding_closed_facts():
    rows, cols = 3, 256
    codes = np.zeros((rows, cols // 2), np.uint8)
    # row 0: inputs j hold q = (j % 16) - 8 (the even input in the low nibble)
    q = (np.arange(cols) % 16) - 8
    codes[0] = ((q[0::2] + 8) | ((q[1::2] + 8) << 4)).astype(np.uint8)
    codes[1] = codes[0]
    codes[2] = codes[0]
    scales = np.zeros((rows, cols // 128), np.uint16)
    scales[0] = bf16_bits([1.0, 1.0])
    scales[1] = bf16_bits([0.125, 4.0])                      # powers of two: exact
    scales[2] = bf16_bits([0.3, -1.7])                       # rounded products
    v = oracle.w4_dequant(codes, scales)
    assert np.array_equal(v[0], q.astype(np.float64))
    assert np.array_equal(v[1, :128], q[:128] * 0.125) and np.array_equal(v[1, 128:], q[128:] * 4.0)
    sc = (scales[2].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = q * np.repeat(sc, 128)
    # nearest bf16 of the exact product: within half a bf16 step (8 significant bits)
    err = np.abs(v[2] - exact)
    assert np.all(err <= np.abs(exact) * 2.0 ** -8 * (1 + 1e-12))
    assert np.array_equal(v[2], loe.bf16_round(exact))
    # the independent numpy decoding agrees bit for bit
    assert np.array_equal(v, loe.w4_dequant_np(codes, scales))


def test_w4_decoding_matches_numpy_on_random_weights():
    rng = np.random.default_rng(21)
    codes = rng.integers(0, 256, (17, 192), dtype=np.uint8)
    scales = bf16_bits(rng.standard_normal((17, 3)).astype(np.float32) * 0.02)
    assert np.array_equal(oracle.w4_dequant(codes, scales), loe.w4_dequant_np(codes, scales))


def test_w4_rejects_ragged_rows():
    with pytest.raises(ValueError):
        oracle.w4_dequant(np.zeros((2, 48), np.uint8), np.zeros((2, 1), np.uint16))


def w4_case(rng, T, d, E, F, *, act, shared=0):
    """Random bf16 x, fp32 router, INT4 experts: uniform codes and bf16 scales
    around 1/(3 sqrt(fan_in)) (so the weights spread like N(0, 1/fan_in))."""
    x32 = rng.standard_normal((T, d)).astype(np.float32)
    x = (x32.view(np.uint32) >> 16).astype(np.uint16)
    Wr = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)
    w = {}

    def mat(rows_shape, fan_in, name):
        w[name] = rng.integers(0, 256, rows_shape + (fan_in // 2,), dtype=np.uint8)
        w[name + "_scale"] = bf16_bits(rng.uniform(0.5, 1.5, rows_shape + (fan_in // 128,)) /
                                       (3.0 * np.sqrt(fan_in)))

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


W4_CASES = [
    dict(act="gelu", score="softmax", renorm=1, k=2, E=6, cap=-1.0, shared=0),
    dict(act="swiglu", score="softmax", renorm=1, k=3, E=8, cap=0.7, shared=0),
    dict(act="swiglu", score="sigmoid", renorm=1, k=4, E=12, cap=-1.0, shared=128),
]


@pytest.mark.parametrize("case", W4_CASES, ids=lambda c: "%s-k%d-cap%s-sh%d" % (
    c["act"], c["k"], c["cap"], c["shared"]))
def test_w4_layer_agrees_with_loop_over_experts(case):
    rng = np.random.default_rng(case["E"] * 3 + case["k"])
    T, d, F = 40, 128, 256
    E, k = case["E"], case["k"]
    x, Wr, w = w4_case(rng, T, d, E, F, act=case["act"], shared=case["shared"])
    sb = rng.normal(0, 0.1, E).astype(np.float32) if case["score"] == "sigmoid" else None
    C = oracle.capacity(case["cap"], k, T, E)
    dims = oracle.make_dims(T, d, E, F, k, x_dtype="bf16", act=case["act"], score=case["score"],
                            renorm=case["renorm"], capacity=C, d_ff_shared=case["shared"])
    r = oracle.route(dims, x, Wr, None, sb)
    dp = oracle.dispatch(dims, r["idx"])
    y = oracle.layer_tokens_w4(dims, x, w, r["idx"], r["gate"], dp["row_of"], np.arange(T))
    ref = loe.layer_w4(x, Wr, w, k, act=case["act"], score=case["score"], renorm=case["renorm"], capacity=C,
                       sel_bias=sb)
    np.testing.assert_array_equal(r["idx"], ref["idx"])
    np.testing.assert_allclose(y, ref["y"], rtol=1e-10, atol=1e-12)


def test_w4_scales_enter_linearly():
    """Doubling every down-projection scale (exact in bf16) doubles the output
    exactly; doubling every up-projection scale doubles H and the output."""
    rng = np.random.default_rng(22)
    T, d, E, F = 6, 128, 2, 128
    x, Wr, w = w4_case(rng, T, d, E, F, act="swiglu")
    dims = oracle.make_dims(T, d, E, F, 1, x_dtype="bf16", act="swiglu")
    tok = np.arange(T, dtype=np.int32)
    ex = np.zeros(T, np.int32)
    base = oracle.expert_apply_w4(dims, x, w, tok, ex)

    def doubled(a):
        return bf16_bits((a.astype(np.uint32) << 16).view(np.float32) * 2.0)

    np.testing.assert_array_equal(oracle.expert_apply_w4(dims, x, dict(w, W2_scale=doubled(w["W2_scale"])), tok, ex),
                                  2.0 * base)
    np.testing.assert_array_equal(oracle.expert_apply_w4(dims, x, dict(w, Wu_scale=doubled(w["Wu_scale"])), tok, ex),
                                  2.0 * base)
