"""Pins of the CPU oracle against what the pages and the mathematics fix.

Nothing here re-types the oracle's formulas: each check is a brute-force
enumeration, a library routine (numpy matmul, scipy softmax / expit / normal
CDF), a closed form the pages state, an invariant, or the second formulation
in oracle/loop_over_experts.py.
"""
import itertools
import json
import os

import numpy as np
import pytest
from scipy import special, stats

import oracle
from oracle import loop_over_experts as loe

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "page_facts.json")


def facts():
    with open(GOLDEN) as f:
        return json.load(f)


def rand_case(rng, T, d, E, d_ff, *, act="gelu", shared=0, bf16=False):
    def mat(*shape, std=1.0):
        a = (rng.standard_normal(shape) * std).astype(np.float32)
        if bf16:
            return (a.view(np.uint32) >> 16).astype(np.uint16)
        return a
    x = mat(T, d)
    Wr = (rng.standard_normal((d, E)) / np.sqrt(d)).astype(np.float32)
    w = dict(W1=mat(E, d_ff, d, std=d ** -0.5), W2=mat(E, d, d_ff, std=d_ff ** -0.5))
    if act == "gelu":
        w["b1"] = rng.uniform(-0.01, 0.01, (E, d_ff)).astype(np.float32)
        w["b2"] = rng.uniform(-0.01, 0.01, (E, d)).astype(np.float32)
    else:
        w["Wu"] = mat(E, d_ff, d, std=d ** -0.5)
    if shared:
        w["Wsg"] = mat(shared, d, std=d ** -0.5)
        w["Wsd"] = mat(d, shared, std=shared ** -0.5)
        if act == "swiglu":
            w["Wsu"] = mat(shared, d, std=d ** -0.5)
    return x, Wr, w


def f64(a):
    return oracle.bf16_bits_to_f64(a)


# --------------------------------------------------------------------------
# top-k selection against brute force
# --------------------------------------------------------------------------
@pytest.mark.parametrize("E", [1, 4, 7, 16])
@pytest.mark.parametrize("score", ["softmax", "sigmoid"])
@pytest.mark.parametrize("biased", [False, True])
def test_topk_matches_brute_force(E, score, biased):
    rng = np.random.default_rng(E * 10 + biased)
    T, d = 24, 12
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    sb = rng.normal(0, 0.3, E).astype(np.float32) if biased else None
    logits = x.astype(np.float64) @ Wr.astype(np.float64)
    for k in range(1, E + 1):
        dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32", score=score)
        r = oracle.route(dims, x, Wr, sel_bias=sb)
        for t in range(T):
            # brute force: score every expert, order all E by (score desc, id asc)
            bias = sb.astype(np.float64) if biased else 0.0
            if score == "softmax":
                # routing score Softmax(W_g x + b) (router-optimization page, How It Works 2)
                key = special.softmax(logits[t] + bias)
            else:
                # selection on sigmoid(logit) + b (auxiliary-loss-free sigmoid routing)
                key = special.expit(logits[t]) + bias
            best = sorted(range(E), key=lambda e: (-key[e], e))[:k]
            assert list(r["idx"][t]) == best, (t, k)


def test_topk_equal_scores_prefer_lower_index():
    # all-equal logits: every order is a tie; the reading picks ascending ids
    T, d, E = 3, 4, 6
    x = np.zeros((T, d), np.float32)
    Wr = np.ones((d, E), np.float32)
    for k in (1, 3, 6):
        r = oracle.route(oracle.make_dims(T, d, E, 8, k, x_dtype="f32"), x, Wr)
        assert (r["idx"] == np.arange(k)[None, :]).all()


# --------------------------------------------------------------------------
# gates
# --------------------------------------------------------------------------
def test_logits_match_library_matmul():
    rng = np.random.default_rng(1)
    T, d, E = 40, 33, 9
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    lb = rng.standard_normal(E).astype(np.float32)
    r = oracle.route(oracle.make_dims(T, d, E, 8, 2, x_dtype="f32"), x, Wr, logit_bias=lb,
                     want_logits=True)
    ref = x.astype(np.float64) @ Wr.astype(np.float64) + lb
    np.testing.assert_allclose(r["logits"], ref, rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("renorm", [0, 1])
def test_softmax_gates(renorm):
    rng = np.random.default_rng(2 + renorm)
    T, d, E, k = 50, 16, 8, 3
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    r = oracle.route(oracle.make_dims(T, d, E, 8, k, x_dtype="f32", renorm=renorm), x, Wr)
    logits = x.astype(np.float64) @ Wr.astype(np.float64)
    p = special.softmax(logits, axis=-1)
    np.testing.assert_allclose(r["pnorm"], p, rtol=1e-13, atol=1e-16)
    sel = np.take_along_axis(logits, r["idx"].astype(np.int64), 1)
    if renorm:
        # softmax over the selected logits (router-optimization formulation)
        np.testing.assert_allclose(r["gate"], special.softmax(sel, axis=-1), rtol=1e-12)
        np.testing.assert_allclose(r["gate"].sum(1), 1.0, rtol=0, atol=1e-12)
    else:
        # gates straight from the full softmax (Eq. moe-output)
        np.testing.assert_allclose(r["gate"], np.take_along_axis(p, r["idx"].astype(np.int64), 1),
                                   rtol=1e-12)
        assert (r["gate"].sum(1) < 1.0).all()


def test_sigmoid_gates_ignore_selection_bias():
    rng = np.random.default_rng(4)
    T, d, E, k = 64, 16, 32, 4
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    sb = rng.normal(0, 0.1, E).astype(np.float32)
    dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32", score="sigmoid")
    r = oracle.route(dims, x, Wr, sel_bias=sb)
    logits = x.astype(np.float64) @ Wr.astype(np.float64)
    s = special.expit(logits)
    sel = np.take_along_axis(s, r["idx"].astype(np.int64), 1)
    np.testing.assert_allclose(r["gate"], sel / sel.sum(1, keepdims=True), rtol=1e-12)
    np.testing.assert_allclose(r["gate"].sum(1), 1.0, atol=1e-12)
    np.testing.assert_allclose(r["pnorm"], s / s.sum(1, keepdims=True), rtol=1e-12)
    # a bias that changes the selection changes which gates appear, but each gate
    # is still the unbiased normalised sigmoid of its expert
    r0 = oracle.route(dims, x, Wr)
    assert (r0["idx"] != r["idx"]).any()


def test_minus_infinity_mask_gives_exact_zero():
    # masking unselected experts before the softmax: those experts get exactly 0
    # weight in the output; with k = E nothing is masked.
    rng = np.random.default_rng(5)
    T, d, E = 10, 8, 5
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    r = oracle.route(oracle.make_dims(T, d, E, 8, E, x_dtype="f32"), x, Wr)
    assert sorted(r["idx"][0]) == list(range(E))
    p = special.softmax(x.astype(np.float64) @ Wr.astype(np.float64), axis=-1)
    np.testing.assert_allclose(np.take_along_axis(p, r["idx"].astype(np.int64), 1), r["gate"], rtol=1e-12)


def test_router_example_shapes():
    fx = facts()["router_example"]
    T = fx["batch"] * fx["seq_len"]
    d, E, k = 64, fx["num_experts"], fx["top_k"]     # d_model shrunk: shapes do not depend on it
    rng = np.random.default_rng(6)
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    r = oracle.route(oracle.make_dims(T, d, E, 8, k, x_dtype="f32"), x, Wr)
    assert list(r["gate"].shape) == fx["weights_shape"]
    assert list(r["idx"].shape) == fx["indices_shape"]


# --------------------------------------------------------------------------
# counts, capacity, permutation
# --------------------------------------------------------------------------
def test_capacity_formula():
    fx = facts()["switch_capacity"]
    assert oracle.capacity(fx["c"], fx["k"], fx["T"], fx["E"]) == fx["capacity"]
    assert oracle.capacity(1.25, 2, 7, 3) == 5          # floor(5.83)
    assert oracle.capacity(1.0, 2, 12, 4) == 6
    assert oracle.capacity(0.0, 2, 12, 4) == -1
    assert oracle.capacity(-1.0, 2, 12, 4) == -1
    u = facts()["uniform_share"]
    assert oracle.capacity(1.0, 1, u["tokens"], u["num_experts"]) == u["per_expert"]


@pytest.mark.parametrize("cap", [-1, 0, 1, 3, 7, 1000])
def test_dispatch_brute_force(cap):
    rng = np.random.default_rng(100 + cap)
    T, E, k = 37, 6, 3
    idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
    dims = oracle.make_dims(T, 8, E, 8, k, x_dtype="f32", capacity=cap)
    dp = oracle.dispatch(dims, idx)
    assert dp["counts"].sum() == T * k
    np.testing.assert_array_equal(dp["counts"], np.bincount(idx.ravel(), minlength=E))
    exp_kept = dp["counts"] if cap < 0 else np.minimum(dp["counts"], cap)
    np.testing.assert_array_equal(dp["kept"], exp_kept)
    assert dp["n_dropped"] == T * k - exp_kept.sum()
    # brute force: list (expert, token) of every assignment, keep the first `cap`
    # tokens of each expert in token order, number the kept ones in (e, t) order
    rows = []
    for e in range(E):
        toks = [t for t in range(T) for s in range(k) if idx[t, s] == e]
        if cap >= 0:
            toks = toks[:cap]
        rows += [(e, t) for t in toks]
    where = {et: i for i, et in enumerate(rows)}
    for t in range(T):
        for s in range(k):
            assert dp["row_of"][t, s] == where.get((int(idx[t, s]), t), -1)
    np.testing.assert_array_equal(dp["row_token"], [t for _, t in rows])
    np.testing.assert_array_equal(dp["offsets"], np.concatenate([[0], np.cumsum(exp_kept)]))


def test_dispatch_rejects_bad_index():
    dims = oracle.make_dims(2, 8, 4, 8, 1, x_dtype="f32")
    with pytest.raises(ValueError):
        oracle.dispatch(dims, np.array([[0], [4]], np.int32))


# --------------------------------------------------------------------------
# balance statistics: closed forms the pages state
# --------------------------------------------------------------------------
@pytest.mark.parametrize("E,k", [(4, 1), (8, 2), (16, 4), (8, 8)])
def test_balance_loss_uniform_is_one(E, k):
    # W_r = [I_E; 0], x_t[:E] = roll(v, t mod E): every expert is chosen equally
    # often and every expert gets the same mean probability.
    d, T = E + 3, 5 * E
    v = np.linspace(2.0, -1.0, E).astype(np.float32)
    x = np.zeros((T, d), np.float32)
    for t in range(T):
        x[t, :E] = np.roll(v, t % E)
    Wr = np.zeros((d, E), np.float32)
    Wr[:E, :E] = np.eye(E, dtype=np.float32)
    dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32")
    r = oracle.route(dims, x, Wr)
    dp = oracle.dispatch(dims, r["idx"])
    b = oracle.balance(dims, dp["counts"], r["pnorm"])
    np.testing.assert_allclose(b["f"], 1.0 / E, rtol=0, atol=1e-15)
    np.testing.assert_allclose(b["P"], 1.0 / E, rtol=1e-13)
    assert abs(b["loss"] - facts()["aux_loss_uniform"]["value"]) < 1e-12


@pytest.mark.parametrize("E", [2, 8, 128])
def test_balance_loss_collapse_is_E(E):
    T, d = 32, 4
    x = np.ones((T, d), np.float32)
    Wr = np.zeros((d, E), np.float32)
    Wr[:, 0] = 25.0                       # logit gap 100 on expert 0
    dims = oracle.make_dims(T, d, E, 8, 1, x_dtype="f32")
    r = oracle.route(dims, x, Wr)
    dp = oracle.dispatch(dims, r["idx"])
    b = oracle.balance(dims, dp["counts"], r["pnorm"])
    assert (r["idx"] == 0).all()
    ratio = facts()["aux_loss_collapse"]["value_over_num_experts"]
    assert abs(b["loss"] / E - ratio) < 1e-12


def test_balance_sigmoid_P_sums_to_one():
    rng = np.random.default_rng(9)
    T, d, E, k = 50, 8, 16, 4
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = rng.standard_normal((d, E)).astype(np.float32)
    dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32", score="sigmoid")
    r = oracle.route(dims, x, Wr)
    b = oracle.balance(dims, oracle.dispatch(dims, r["idx"])["counts"], r["pnorm"])
    assert abs(b["P"].sum() - 1.0) < 1e-12
    assert abs(b["f"].sum() - 1.0) < 1e-12


def test_active_fraction_facts():
    for E, k, frac in facts()["active_fraction"]["cases"]:
        rng = np.random.default_rng(E)
        T, d = 30, 6
        x = rng.standard_normal((T, d)).astype(np.float32)
        Wr = rng.standard_normal((d, E)).astype(np.float32)
        dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32")
        r = oracle.route(dims, x, Wr)
        active = np.array([len(set(row)) for row in r["idx"]]) / E
        np.testing.assert_allclose(active, frac, atol=5e-4)


# --------------------------------------------------------------------------
# expert FFN and layer output
# --------------------------------------------------------------------------
@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_single_expert_is_dense_ffn(act):
    # E = 1, k = 1, renormalised gate = 1: the layer is one dense FFN
    rng = np.random.default_rng(11)
    T, d, F = 9, 24, 40
    x, Wr, w = rand_case(rng, T, d, 1, F, act=act)
    dims = oracle.make_dims(T, d, 1, F, 1, x_dtype="f32", act=act)
    out = oracle.forward(dims, x, Wr, w)
    xf = x.astype(np.float64)
    if act == "gelu":
        a = xf @ w["W1"][0].astype(np.float64).T + w["b1"][0]
        ref = (a * stats.norm.cdf(a)) @ w["W2"][0].astype(np.float64).T + w["b2"][0]
    else:
        g = xf @ w["W1"][0].astype(np.float64).T
        u = xf @ w["Wu"][0].astype(np.float64).T
        ref = (g * special.expit(g) * u) @ w["W2"][0].astype(np.float64).T
    np.testing.assert_allclose(out["gate"], 1.0, rtol=0, atol=1e-15)
    np.testing.assert_allclose(out["y"], ref, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("act", ["gelu", "swiglu"])
def test_k_equals_E_is_full_soft_mixture(act):
    # k = E without renormalisation: y = sum_e softmax(h)_e * E_e(x)
    rng = np.random.default_rng(12)
    T, d, E, F = 11, 16, 5, 24
    x, Wr, w = rand_case(rng, T, d, E, F, act=act)
    dims = oracle.make_dims(T, d, E, F, E, x_dtype="f32", act=act, renorm=0)
    out = oracle.forward(dims, x, Wr, w)
    xf = x.astype(np.float64)
    p = special.softmax(xf @ Wr.astype(np.float64), axis=-1)
    ref = np.zeros((T, d))
    for e in range(E):
        if act == "gelu":
            a = xf @ w["W1"][e].astype(np.float64).T + w["b1"][e]
            o = (a * stats.norm.cdf(a)) @ w["W2"][e].astype(np.float64).T + w["b2"][e]
        else:
            g = xf @ w["W1"][e].astype(np.float64).T
            u = xf @ w["Wu"][e].astype(np.float64).T
            o = (g * special.expit(g) * u) @ w["W2"][e].astype(np.float64).T
        ref += p[:, e:e + 1] * o
    np.testing.assert_allclose(out["y"], ref, rtol=1e-11, atol=1e-12)


CASES = [
    dict(act="gelu", score="softmax", renorm=1, k=2, E=8, cap=-1.0, shared=0),
    dict(act="gelu", score="softmax", renorm=0, k=1, E=6, cap=1.25, shared=0),
    dict(act="swiglu", score="softmax", renorm=1, k=3, E=9, cap=-1.0, shared=0),
    dict(act="swiglu", score="softmax", renorm=1, k=2, E=4, cap=0.6, shared=0),
    dict(act="swiglu", score="sigmoid", renorm=1, k=4, E=16, cap=-1.0, shared=24),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "%s-%s-k%d-cap%s-sh%d" % (
    c["act"], c["score"], c["k"], c["cap"], c["shared"]))
@pytest.mark.parametrize("bf16", [False, True])
def test_oracle_agrees_with_loop_over_experts(case, bf16):
    rng = np.random.default_rng(hash((case["act"], case["k"], case["E"], bf16)) & 0xFFFF)
    T, d, F = 45, 32, 48
    E, k = case["E"], case["k"]
    x, Wr, w = rand_case(rng, T, d, E, F, act=case["act"], shared=case["shared"], bf16=bf16)
    lb = rng.normal(0, 1, E).astype(np.float32)
    sb = rng.normal(0, 0.1, E).astype(np.float32) if case["score"] == "sigmoid" else None
    C = oracle.capacity(case["cap"], k, T, E)
    dims = oracle.make_dims(T, d, E, F, k, x_dtype="bf16" if bf16 else "f32", act=case["act"],
                            score=case["score"], renorm=case["renorm"], capacity=C,
                            d_ff_shared=case["shared"])
    out = oracle.forward(dims, x, Wr, w, logit_bias=lb, sel_bias=sb)
    ref = loe.layer(x, Wr, w, k, act=case["act"], score=case["score"], renorm=case["renorm"],
                    capacity=C, logit_bias=lb, sel_bias=sb)
    np.testing.assert_array_equal(out["idx"], ref["idx"])
    np.testing.assert_allclose(out["gate"], ref["gate"], rtol=1e-12)
    np.testing.assert_array_equal(out["counts"], ref["counts"])
    np.testing.assert_array_equal(out["kept"], ref["kept"])
    rows = [(e, t) for e in range(E) for t in out["row_token"][out["offsets"][e]:out["offsets"][e + 1]]]
    assert rows == ref["perm_rows"]
    np.testing.assert_allclose(out["y"], ref["y"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(out["f"], ref["f"], rtol=1e-14)
    np.testing.assert_allclose(out["P"], ref["P"], rtol=1e-12)
    assert abs(out["loss"] - ref["loss"]) < 1e-12 * max(1.0, abs(ref["loss"]))
    if C >= 0 and out["n_dropped"]:
        # a dropped assignment contributes nothing: zero every dropped slot's gate
        # and the output must not move
        g2 = out["gate"].copy()
        g2[out["row_of"] < 0] = 0.0
        y2 = oracle.layer_tokens(dims, x, w, out["idx"], g2, None, out["tokens"])
        np.testing.assert_allclose(y2, out["y"], rtol=1e-13, atol=1e-15)


def test_bf16_inputs_widen_exactly():
    rng = np.random.default_rng(13)
    T, d, E, F = 7, 16, 4, 16
    xb, Wr, wb = rand_case(rng, T, d, E, F, act="swiglu", bf16=True)
    wf = {k2: (f64(v).astype(np.float32) if v.dtype == np.uint16 else v) for k2, v in wb.items()}
    xf = f64(xb).astype(np.float32)
    db = oracle.make_dims(T, d, E, F, 2, x_dtype="bf16", act="swiglu")
    df = oracle.make_dims(T, d, E, F, 2, x_dtype="f32", act="swiglu")
    yb = oracle.forward(db, xb, Wr, wb)["y"]
    yf = oracle.forward(df, xf, Wr, wf)["y"]
    np.testing.assert_array_equal(yb, yf)


def test_expert_apply_matches_layer_sum():
    rng = np.random.default_rng(14)
    T, d, E, F, k = 12, 16, 6, 24, 2
    x, Wr, w = rand_case(rng, T, d, E, F, act="swiglu", shared=16)
    dims = oracle.make_dims(T, d, E, F, k, x_dtype="f32", act="swiglu", d_ff_shared=16)
    out = oracle.forward(dims, x, Wr, w)
    tok = np.repeat(np.arange(T), k)
    rows = oracle.expert_apply(dims, x, w, tok, out["idx"].ravel(), out["gate"].ravel())
    sh = oracle.expert_apply(dims, x, w, np.arange(T), np.full(T, E))
    y = rows.reshape(T, k, d).sum(1) + sh
    np.testing.assert_allclose(y, out["y"], rtol=1e-12, atol=1e-14)
    with pytest.raises(ValueError):
        oracle.expert_apply(dims, x, w, [0], [E + 1])


# --------------------------------------------------------------------------
# auxiliary-loss-free bias update and routing health
# --------------------------------------------------------------------------
def test_bias_update_follows_the_sign_rule():
    fx = facts()["bias_rule"]
    gamma = fx["gamma"]
    T, k, E = 12, 2, 4                      # target load T k / E = 6
    dims = oracle.make_dims(T, 8, E, 8, k, x_dtype="f32")
    counts = np.array([9, 6, 3, 6], np.int32)
    b0 = np.array([0.5, -0.25, 0.0, 1.0], np.float32)
    b1 = oracle.bias_update(dims, counts, b0, gamma)
    # overloaded expert 0 loses gamma, underloaded expert 2 gains it, exactly
    # loaded experts 1 and 3 keep their bias
    np.testing.assert_array_equal(b1, np.array([0.5 - gamma, -0.25, 0.0 + gamma, 1.0], np.float32))
    np.testing.assert_array_equal(b0, [0.5, -0.25, 0.0, 1.0])      # input untouched


def test_bias_update_balances_a_skewed_router():
    # repeated updates on a fixed, skewed router move load off the hot expert
    rng = np.random.default_rng(21)
    T, d, E, k = 256, 16, 8, 2
    x = rng.standard_normal((T, d)).astype(np.float32)
    Wr = (rng.standard_normal((d, E)) * 0.3).astype(np.float32)
    lb = np.array([2.0, 1.0] + [0.0] * (E - 2), np.float32)
    dims = oracle.make_dims(T, d, E, 8, k, x_dtype="f32", score="sigmoid")
    b = np.zeros(E, np.float32)
    first = None
    for _ in range(400):
        r = oracle.route(dims, x, Wr, lb, b, want_pnorm=False)
        counts = oracle.dispatch(dims, r["idx"])["counts"]
        if first is None:
            first = counts.max() / (T * k / E)
        b = oracle.bias_update(dims, counts, b, 0.01)
    last = counts.max() / (T * k / E)
    assert first > 2.0 and last < first / 1.5


def test_routing_health_closed_forms():
    E = facts()["entropy_max_128"]["num_experts"]
    T, k = 256, 2
    dims = oracle.make_dims(T, 8, E, 8, k, x_dtype="f32")
    uniform = oracle.routing_health(dims, np.full(E, T * k // E, np.int32), np.full(E, 1.0 / E))
    assert abs(uniform["entropy"] - np.log(E)) < 1e-12
    assert round(uniform["entropy"], facts()["entropy_max_128"]["printed_digits"]) == facts()["entropy_max_128"]["value"]
    assert uniform["ratio"] == 1.0 and abs(uniform["max_share"] - 1.0 / E) < 1e-15
    onehot_P = np.zeros(E); onehot_P[3] = 1.0
    counts = np.zeros(E, np.int32); counts[3] = T * k
    collapsed = oracle.routing_health(dims, counts, onehot_P)
    assert collapsed["entropy"] == 0.0 and collapsed["ratio"] == float("inf") and collapsed["max_share"] == 1.0
    # a 2:1 split of the load between two halves of the experts
    c = np.array([2] * (E // 2) + [1] * (E // 2), np.int32) * 4
    h = oracle.routing_health(dims, c, c / c.sum())
    assert h["ratio"] == 2.0
    assert abs(h["entropy"] - stats.entropy(c / c.sum())) < 1e-12   # scipy's Shannon entropy
