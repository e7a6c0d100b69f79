"""Pins of the oracle's backward pass (CPU): central finite differences of the
oracle's own forward pass, which is pinned independently
(test_oracle_pins.py).

ell = sum_t <dy_t, y_t> + alpha * L_aux is evaluated with oracle.forward
(fp64 arithmetic on fp32 inputs).  Each input coordinate v is moved to
v +- 2^-10, a step that keeps v exactly representable in fp32 (|v| < 2^13),
and (ell(v + h) - ell(v - h)) / 2h must match the oracle_layer_backward
gradient: the central difference is exact up to h^2 times a third
derivative (about 1e-6 here), so the bound is 2e-5 of the parameter's
largest gradient entry plus 1e-7.  Inputs are redrawn until every token's
selection margin is at least 0.05, so no step of 2^-10 changes which experts
are chosen or dropped (the gradient of that piecewise-constant choice is
zero by definition).  Every variant of the layer is covered: renormalised and
full-softmax gates, sigmoid gates with a selection bias, GELU experts with
biases, SwiGLU experts, capacity drops, a shared expert, the logit offset and
the aux-loss term alone.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import enforce_margin, oracle_dims, to_host

H = 2.0 ** -10
W = syn.Workload
WEIGHTS = ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd")

CASES = [
    (W("swiglu_renorm", T=7, d_model=8, E=4, d_ff=6, top_k=2, dtype="f32", logit_skew="normal"), 0.7),
    (W("gelu_full_softmax_cap", T=9, d_model=6, E=4, d_ff=5, top_k=2, dtype="f32", act="gelu", renorm=0,
       capacity_factor=0.6, logit_skew="normal"), 0.3),
    (W("sigmoid_bias_shared", T=6, d_model=8, E=5, d_ff=4, top_k=2, dtype="f32", score="sigmoid",
       sel_bias_std=0.2, d_ff_shared=6), 0.5),
    (W("gelu_renorm_shared_k3", T=5, d_model=6, E=4, d_ff=4, top_k=3, dtype="f32", act="gelu",
       d_ff_shared=5), 1.0),
]


def make(wl, seed):
    inp = syn.generate(wl, "cpu", seed)
    host = to_host(inp)
    enforce_margin(wl, inp, host, seed, margin=0.05)
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal((wl.T, wl.d_model))
    return host, dy


def loss(dims, host, dy, alpha):
    w = {k: host[k] for k in WEIGHTS if host.get(k) is not None}
    out = oracle.forward(dims, host["x"], host["Wr"], w, logit_bias=host.get("logit_bias"),
                         sel_bias=host.get("sel_bias"))
    return float(np.sum(dy * out["y"]) + alpha * out["loss"])


def grads(dims, host, dy, alpha):
    w = {k: host[k] for k in WEIGHTS if host.get(k) is not None}
    return oracle.layer_backward(dims, host["x"], host["Wr"], w, dy, alpha, logit_bias=host.get("logit_bias"),
                                 sel_bias=host.get("sel_bias"))


GRAD_OF = {"x": "dx", "Wr": "dWr", "logit_bias": "dbeta", "W1": "dW1", "Wu": "dWu", "W2": "dW2", "b1": "db1",
           "b2": "db2", "Wsg": "dWsg", "Wsu": "dWsu", "Wsd": "dWsd"}


def fd_check(wl, host, dy, alpha, max_coords=60, seed=0):
    dims = oracle_dims(wl)
    g = grads(dims, host, dy, alpha)
    rng = np.random.default_rng(seed)
    checked = 0
    for name, gname in GRAD_OF.items():
        v = host.get(name)
        if v is None:
            continue
        gv = g[gname]
        assert gv is not None and gv.shape == v.shape, name
        flat = v.reshape(-1)
        coords = rng.choice(flat.size, size=min(max_coords, flat.size), replace=False)
        bound = 2e-5 * np.max(np.abs(gv)) + 1e-7
        for c in coords:
            orig = flat[c]
            assert abs(orig) < 2.0 ** 13
            flat[c] = np.float32(orig + H)
            lp = loss(dims, host, dy, alpha)
            flat[c] = np.float32(orig - H)
            lm = loss(dims, host, dy, alpha)
            flat[c] = orig
            fd = (lp - lm) / (2 * H)
            assert abs(fd - gv.reshape(-1)[c]) <= bound, (name, int(c), fd, gv.reshape(-1)[c])
            checked += 1
    return g, checked


@pytest.mark.parametrize("wl,alpha", CASES, ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_backward_matches_finite_differences(wl, alpha):
    host, dy = make(wl, seed=3)
    g, n = fd_check(wl, host, dy, alpha)
    assert n > 100


def test_aux_loss_gradient_alone():
    # dy = 0: only alpha * L_aux remains; its gradient reaches the router
    # (x through W_r, W_r, the logit offset) and no expert weight
    wl, _ = CASES[0]
    host, _ = make(wl, seed=4)
    dy = np.zeros((wl.T, wl.d_model))
    g, _ = fd_check(wl, host, dy, alpha=2.0)
    for name in ("dW1", "dWu", "dW2"):
        assert np.all(g[name] == 0.0)
    assert np.max(np.abs(g["dWr"])) > 0 and np.max(np.abs(g["dbeta"])) > 0
    # the aux term is E * sum_e f_e P_e with sum_e P_e = 1 for every token: the
    # logit-offset gradient sums to zero over experts
    assert abs(np.sum(g["dbeta"])) < 1e-12


def test_dropped_slots_carry_no_gradient():
    # with capacity 0.6 some assignments are dropped; an expert that kept no
    # row gets exactly zero weight gradient
    wl, alpha = CASES[1]
    host, dy = make(wl, seed=5)
    dims = oracle_dims(wl)
    r = oracle.route(dims, host["x"], host["Wr"], host.get("logit_bias"))
    dp = oracle.dispatch(dims, r["idx"])
    assert dp["n_dropped"] > 0
    g = grads(dims, host, dy, alpha)
    for e in range(wl.E):
        if dp["kept"][e] == 0:
            assert np.all(g["dW1"][e] == 0) and np.all(g["dW2"][e] == 0) and np.all(g["db1"][e] == 0)


def test_dense_ffn_special_case_matches_autograd():
    # E = 1, k = 1: a dense SwiGLU FFN with gate 1.  Its gradients from the
    # oracle equal those of the same dense FFN written as torch operations in
    # float64 and differentiated by autograd (an independent derivative)
    wl = W("dense", T=5, d_model=8, E=1, d_ff=6, top_k=1, dtype="f32")
    host, dy = make(wl, seed=6)
    dims = oracle_dims(wl)
    g = grads(dims, host, dy, alpha=0.0)
    x = torch.tensor(host["x"], dtype=torch.float64, requires_grad=True)
    Wg = torch.tensor(host["W1"][0], dtype=torch.float64, requires_grad=True)
    Wu = torch.tensor(host["Wu"][0], dtype=torch.float64, requires_grad=True)
    Wd = torch.tensor(host["W2"][0], dtype=torch.float64, requires_grad=True)
    y = (torch.nn.functional.silu(x @ Wg.T) * (x @ Wu.T)) @ Wd.T
    (y * torch.tensor(dy)).sum().backward()
    np.testing.assert_allclose(g["dW1"][0], Wg.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dWu"][0], Wu.grad.numpy(), rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(g["dW2"][0], Wd.grad.numpy(), rtol=1e-12, atol=1e-14)
    # the router sees no gradient: a single expert's gate is 1 whatever h is
    np.testing.assert_allclose(g["dx"], x.grad.numpy(), rtol=1e-12, atol=1e-14)
    assert np.all(np.abs(g["dWr"]) < 1e-15)
