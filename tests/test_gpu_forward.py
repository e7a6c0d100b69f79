"""GPU parity of the whole layer (moe_forward through the C ABI) against the
CPU oracle on the same seeded inputs.

Routing (expert ids, counts, capacity drops) and the dispatch tables the
forward pass leaves in its workspace (kept, offsets, row_of, row_token: the
(expert, token) row order) must match bit for bit; gates to 1e-5; the output
to max|y - y_ref| / max|y_ref| <= 2e-2 for bf16 layers and 1e-4 for fp32
layers; the balance loss to 1e-5 relative.  Small cases are checked on every
token.  The five full-size workloads run in the benchmark's launch
configuration: routing, dispatch tables and loss over all tokens; y over all
tokens for the fp32, Switch- and Qwen3-shaped layers and over 2048 sampled
tokens plus one token of every expert that kept a row for the Mixtral- and
DeepSeek-shaped layers (whose fp64 oracle costs about 0.7 GFLOP per token).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import (TOL_BF16, TOL_F32, TOL_LOGIT, TOL_LOSS, check_routing, make_case, oracle_dims, rel_err,
                     sample_tokens, to_f64, weights_host)

pytestmark = pytest.mark.gpu

W = syn.Workload


def run_forward(wl, inp, want_logits=False):
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, want_logits=want_logits)
    ws = nat.alloc_workspace(cfg)
    nat.forward(cfg, inp, out, ws)
    status = nat.moe_get_device_status(ws)
    assert status == nat.MOE_OK, nat.status_string(status)
    return cfg, out, ws


def check_forward(wl, inp, host, n_sample=None, seed=0):
    cfg, out, ws = run_forward(wl, inp, want_logits=True)
    dims = oracle_dims(wl)
    r = oracle.route(dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"], want_logits=True)
    dp = oracle.dispatch(dims, r["idx"])
    bal = oracle.balance(dims, dp["counts"], r["pnorm"])

    gpu_idx = out.idx.cpu().numpy()
    swapped = check_routing(gpu_idx, out.gate.cpu().numpy(), r)
    np.testing.assert_array_equal(out.counts.cpu().numpy(), dp["counts"])
    assert int(out.n_dropped.item()) == dp["n_dropped"]
    # the forward pass's dispatch tables against the oracle's dispatch of the
    # same expert ids (slot order may differ from the oracle's only between
    # tied keys; the tables of a given selection are unique)
    dpg = dp if swapped == 0 else oracle.dispatch(dims, gpu_idx)
    tab = nat.workspace_tables(cfg, ws)
    nrows = int(dpg["offsets"][-1])
    np.testing.assert_array_equal(tab["kept"].cpu().numpy(), dpg["kept"])
    np.testing.assert_array_equal(tab["offsets"].cpu().numpy(), dpg["offsets"])
    np.testing.assert_array_equal(tab["row_of"].cpu().numpy(), dpg["row_of"])
    np.testing.assert_array_equal(tab["row_token"][:nrows].cpu().numpy(), dpg["row_token"])
    # each row carries its assignment's gate, bit for bit
    ro = dpg["row_of"]
    kept_slots = ro >= 0
    np.testing.assert_array_equal(tab["row_gate"][:nrows].cpu().numpy()[ro[kept_slots]],
                                  out.gate.cpu().numpy()[kept_slots])
    assert rel_err(out.logits.cpu().numpy(), r["logits"]) < TOL_LOGIT
    loss = float(out.loss.item())
    assert abs(loss - bal["loss"]) <= TOL_LOSS * abs(bal["loss"])
    np.testing.assert_allclose(out.f.cpu().numpy(), bal["f"], rtol=1e-6)
    np.testing.assert_allclose(out.P.cpu().numpy(), bal["P"], rtol=1e-4, atol=1e-7)

    if n_sample is None:
        tokens = np.arange(wl.T, dtype=np.int32)
    else:
        tokens = sample_tokens(r["idx"], dp["row_of"], wl.E, n_sample, seed, wl.T)
    y_ref = oracle.layer_tokens(dims, host["x"], weights_host(host), r["idx"], r["gate"], dp["row_of"], tokens)
    y = to_f64(out.y)[tokens]
    err = rel_err(y, y_ref)
    tol = TOL_F32 if wl.dtype == "f32" else TOL_BF16
    assert err <= tol, "max|y-y_ref|/max|y_ref| = %.3e > %.1e" % (err, tol)
    return dict(err=err, loss=loss, loss_ref=bal["loss"], out=out, ref=r, dp=dp, tokens=tokens, swapped=swapped)


SMALL = [
    W("tiny_fp32", T=256, d_model=128, E=8, d_ff=256, top_k=2, dtype="f32", act="gelu"),
    W("f32_swiglu_shared", T=150, d_model=96, E=6, d_ff=80, top_k=2, dtype="f32", d_ff_shared=48,
      score="sigmoid", sel_bias_std=0.1),
    W("switch_small", T=600, d_model=256, E=16, d_ff=384, top_k=1, act="gelu", renorm=0,
      capacity_factor=1.25, logit_skew="normal"),
    W("mixtral_small", T=520, d_model=384, E=8, d_ff=448, top_k=2),
    W("qwen_small", T=700, d_model=256, E=32, d_ff=192, top_k=8, logit_skew="zipf"),
    W("deepseek_small", T=333, d_model=512, E=64, d_ff=256, top_k=8, score="sigmoid",
      d_ff_shared=384, sel_bias_std=0.1),
    W("ragged_widths", T=301, d_model=200, E=5, d_ff=136, top_k=2, act="gelu", d_ff_shared=72),
    W("dense_single_expert", T=257, d_model=128, E=1, d_ff=256, top_k=1),
    W("soft_mixture_k_eq_E", T=130, d_model=128, E=4, d_ff=128, top_k=4, renorm=0, act="gelu"),
    W("tight_capacity", T=400, d_model=128, E=8, d_ff=128, top_k=2, capacity_factor=0.3,
      logit_skew="normal"),
    # selection edge cases: every lane keeps a slot (k = 32); eight candidates
    # per lane with softmax scores (E = 256)
    W("k32", T=160, d_model=128, E=64, d_ff=128, top_k=32),
    W("e256_softmax", T=300, d_model=256, E=256, d_ff=64, top_k=4, logit_skew="normal"),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_forward_small(wl, cuda_device):
    inp, host = make_case(wl, cuda_device, seed=1)
    check_forward(wl, inp, host)


# y checked on every token (None) or on this many sampled tokens plus one
# token of every expert that kept a row
FULL_SIZE_Y_TOKENS = {"tiny_fp32": None, "switch_top1": None, "qwen3_moe": None, "mixtral": 2048,
                      "deepseek_v3": 2048}


@pytest.mark.parametrize("name", ["tiny_fp32", "switch_top1", "mixtral", "qwen3_moe", "deepseek_v3"])
def test_forward_full_size(name, cuda_device):
    wl = syn.WORKLOADS[name]
    inp, host = make_case(wl, cuda_device, seed=0)
    res = check_forward(wl, inp, host, n_sample=FULL_SIZE_Y_TOKENS[name])
    print("%s: max rel err %.3e, loss %.6f (ref %.6f), %d tokens checked, %d tie-swapped slot orders" % (
        name, res["err"], res["loss"], res["loss_ref"], len(res["tokens"]), res["swapped"]))


def test_forward_long_sequence(cuda_device):
    # T = 20000 tokens: 313 dispatch chunks, so the per-expert scan over chunks
    # takes two passes (256 chunks each); tight capacity drops assignments
    wl = W("long_T", T=20000, d_model=128, E=16, d_ff=128, top_k=2, capacity_factor=0.9, logit_skew="normal")
    inp, host = make_case(wl, cuda_device, seed=2)
    res = check_forward(wl, inp, host)
    assert res["dp"]["n_dropped"] > 0


def test_forward_is_deterministic(cuda_device):
    wl = W("det", T=700, d_model=256, E=32, d_ff=192, top_k=8, logit_skew="zipf", d_ff_shared=128)
    inp, _ = make_case(wl, cuda_device, seed=3)
    _, a, _ = run_forward(wl, inp)
    _, b, _ = run_forward(wl, inp)
    assert torch.equal(a.y, b.y) and torch.equal(a.idx, b.idx) and torch.equal(a.gate, b.gate)
    assert torch.equal(a.loss, b.loss) and torch.equal(a.P, b.P)


def test_uniform_routing_gives_loss_one(cuda_device):
    # W_r = [I_E; 0] and x_t[:E] = roll(v, t mod E): f_e = P_e = 1/E, L = 1
    E, k, d, F = 16, 4, 64, 128
    T = 8 * E
    wl = W("uniform", T=T, d_model=d, E=E, d_ff=F, top_k=k, dtype="f32")
    inp = syn.generate(wl, cuda_device, seed=0)
    v = torch.linspace(2.0, -1.0, E)
    x = torch.zeros((T, d))
    for t in range(T):
        x[t, :E] = torch.roll(v, t % E)
    Wr = torch.zeros((d, E))
    Wr[:E, :E] = torch.eye(E)
    inp["x"] = x.to(cuda_device)
    inp["Wr"] = Wr.to(cuda_device)
    _, out, _ = run_forward(wl, inp)
    assert abs(float(out.loss.item()) - 1.0) < 1e-5
    assert torch.all(out.counts == T * k // E)


def test_collapse_gives_loss_E(cuda_device):
    E = 8
    wl = W("collapse", T=64, d_model=64, E=E, d_ff=128, top_k=1, dtype="f32")
    inp = syn.generate(wl, cuda_device, seed=0)
    inp["x"] = torch.ones((64, 64), device=cuda_device)
    Wr = torch.zeros((64, E))
    Wr[:, 3] = 100.0 / 64
    inp["Wr"] = Wr.to(cuda_device)
    _, out, _ = run_forward(wl, inp)
    assert torch.all(out.idx == 3)
    assert abs(float(out.loss.item()) / E - 1.0) < 1e-5


@pytest.mark.parametrize("cap", [0.0, 0.5])
def test_all_tokens_one_expert_bf16(cap, cuda_device):
    # every token picks expert 2 first: one expert holds T rows (several tiles),
    # with a capacity limit most of them are dropped
    wl = W("hot_expert", T=1000, d_model=128, E=4, d_ff=256, top_k=2, capacity_factor=cap)
    inp, host = make_case(wl, cuda_device, seed=5)
    lb = torch.tensor([0.0, 0.0, 30.0, 0.0], device=cuda_device)
    inp["logit_bias"] = lb
    host["logit_bias"] = lb.cpu().numpy()
    from helpers import enforce_margin
    enforce_margin(wl, inp, host, seed=5)
    res = check_forward(wl, inp, host)
    assert (res["ref"]["idx"][:, 0] == 2).all()


@pytest.mark.parametrize("T", [0, 1, 2, 33])
def test_forward_tiny_T(T, cuda_device):
    wl = W("tinyT", T=T, d_model=64, E=8, d_ff=128, top_k=2, d_ff_shared=64)
    inp, host = make_case(wl, cuda_device, seed=7)
    if T == 0:
        cfg, out, _ = run_forward(wl, inp)
        assert out.y.numel() == 0
        assert int(out.counts.sum().item()) == 0
        assert np.isnan(float(out.loss.item()))
    else:
        check_forward(wl, inp, host)
