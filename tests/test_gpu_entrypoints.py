"""GPU parity of each C-ABI entry point on its own, against the oracle.

moe_router_topk:   ids bit-exact, gates 1e-5, logits 1e-5 relative, P from psum
moe_permute:       counts / kept / offsets / row_of / row_token bit-exact,
                   x_perm rows equal the source rows, row_gate the gates
moe_grouped_ffn:   every packed row against the oracle expert applied to its
                   token and scaled by its gate
moe_combine:       the gather-sum against a float64 sum of the same rows
moe_balance_stats: f, P, loss against the oracle
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import (TOL_BF16, TOL_F32, TOL_LOGIT, TOL_LOSS, check_routing, make_case, oracle_dims, rel_err,
                     to_f64, weights_host)

pytestmark = pytest.mark.gpu

W = syn.Workload
CASES = [
    W("swiglu_cap", T=900, d_model=256, E=12, d_ff=320, top_k=3, capacity_factor=0.9, logit_skew="normal"),
    W("gelu_f32", T=300, d_model=64, E=8, d_ff=96, top_k=2, dtype="f32", act="gelu"),
    W("sigmoid_shared", T=500, d_model=192, E=40, d_ff=128, top_k=6, score="sigmoid",
      sel_bias_std=0.1, d_ff_shared=256),
]


class Stage:
    """Runs the layer entry point by entry point, keeping every intermediate."""

    def __init__(self, wl, inp):
        dev = inp["x"].device
        self.cfg = cfg = nat.config_from_workload(wl)
        T, d, E, k = wl.T, wl.d_model, wl.E, wl.top_k
        dt = nat.layer_dtype(cfg)
        self.ws = nat.alloc_workspace(cfg, dev)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.gate = torch.empty((T, k), dtype=torch.float32, device=dev)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=dev)
        self.psum = torch.empty((nat.router_blocks(cfg), E), dtype=torch.float32, device=dev)
        self.counts = torch.empty(E, dtype=torch.int32, device=dev)
        self.kept = torch.empty(E, dtype=torch.int32, device=dev)
        self.offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
        self.row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
        self.row_token = torch.full((T * k,), -1, dtype=torch.int32, device=dev)
        self.row_gate = torch.zeros(T * k, dtype=torch.float32, device=dev)
        self.x_perm = torch.zeros((T * k, d), dtype=dt, device=dev)
        self.n_dropped = torch.zeros(1, dtype=torch.int32, device=dev)
        self.y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=dt, device=dev)
        self.y = torch.empty((T, d), dtype=dt, device=dev)
        self.f = torch.empty(E, dtype=torch.float32, device=dev)
        self.P = torch.empty(E, dtype=torch.float32, device=dev)
        self.loss = torch.empty(1, dtype=torch.float64, device=dev)
        self.inp = inp

    def router(self):
        i = self.inp
        nat.moe_router_topk(self.cfg, i["x"], i["Wr"], i["logit_bias"], i["sel_bias"], self.idx, self.gate,
                            self.logits, self.psum, self.ws)

    def permute(self):
        nat.moe_permute(self.cfg, self.inp["x"], self.idx, self.gate, self.counts, self.kept, self.offsets,
                        self.row_of, self.row_token, self.row_gate, self.x_perm, self.n_dropped, self.ws)

    def ffn(self):
        i = self.inp
        nat.moe_grouped_ffn(self.cfg, self.x_perm, self.offsets, self.row_gate, i["W1"], i["b1"], i["Wu"], i["W2"],
                            i["b2"], i["x"], i["Wsg"], i["Wsu"], i["Wsd"], self.y_perm, self.ws)

    def combine(self):
        nat.moe_combine(self.cfg, self.y_perm, self.row_of, self.y, self.ws)

    def balance(self):
        nat.moe_balance_stats(self.cfg, self.counts, self.psum, self.f, self.P, self.loss)

    def status(self):
        return nat.moe_get_device_status(self.ws)


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_entry_points(wl, cuda_device):
    inp, host = make_case(wl, cuda_device, seed=11)
    dims = oracle_dims(wl)
    st = Stage(wl, inp)
    T, k, E = wl.T, wl.top_k, wl.E

    # ---- router
    st.router()
    assert st.status() == nat.MOE_OK
    r = oracle.route(dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"], want_logits=True)
    check_routing(st.idx.cpu().numpy(), st.gate.cpu().numpy(), r)
    assert rel_err(st.logits.cpu().numpy(), r["logits"]) < TOL_LOGIT
    P_gpu = st.psum.double().sum(0).cpu().numpy() / T
    np.testing.assert_allclose(P_gpu, r["pnorm"].mean(0), rtol=1e-4, atol=1e-7)

    # ---- permute (compare on the GPU's own ids, which equal the oracle's)
    st.permute()
    assert st.status() == nat.MOE_OK
    dp = oracle.dispatch(dims, st.idx.cpu().numpy())
    np.testing.assert_array_equal(st.counts.cpu().numpy(), dp["counts"])
    np.testing.assert_array_equal(st.kept.cpu().numpy(), dp["kept"])
    np.testing.assert_array_equal(st.offsets.cpu().numpy(), dp["offsets"])
    np.testing.assert_array_equal(st.row_of.cpu().numpy(), dp["row_of"])
    nrows = int(dp["offsets"][-1])
    np.testing.assert_array_equal(st.row_token[:nrows].cpu().numpy(), dp["row_token"])
    assert int(st.n_dropped.item()) == dp["n_dropped"]
    rt = st.row_token[:nrows].long()
    assert torch.equal(st.x_perm[:nrows], inp["x"][rt])
    g = st.gate.cpu().numpy()
    ro = dp["row_of"]
    exp_gate = np.zeros(nrows, np.float32)
    for t in range(T):
        for s in range(k):
            if ro[t, s] >= 0:
                exp_gate[ro[t, s]] = g[t, s]
    np.testing.assert_array_equal(st.row_gate[:nrows].cpu().numpy(), exp_gate)
    # without x_perm the same row tables come out and nothing else is written
    rt2 = torch.full_like(st.row_token, -7)
    ro2 = torch.full_like(st.row_of, -7)
    rg2 = torch.zeros_like(st.row_gate)
    nat.moe_permute(st.cfg, inp["x"], st.idx, st.gate, st.counts, st.kept, st.offsets, ro2, rt2, rg2, None,
                    st.n_dropped, st.ws)
    assert st.status() == nat.MOE_OK
    assert torch.equal(ro2, st.row_of) and torch.equal(rt2[:nrows], st.row_token[:nrows])
    assert torch.equal(rg2[:nrows], st.row_gate[:nrows])

    # ---- grouped FFN: each packed row against the oracle expert on its token
    st.ffn()
    assert st.status() == nat.MOE_OK
    row_expert = np.repeat(np.arange(E), dp["kept"]).astype(np.int32)
    tok = dp["row_token"]
    tol = TOL_F32 if wl.dtype == "f32" else TOL_BF16
    ref_rows = oracle.expert_apply(dims, host["x"], weights_host(host), tok, row_expert,
                                   st.row_gate[:nrows].double().cpu().numpy())
    got_rows = to_f64(st.y_perm[:nrows])
    for e in range(E):
        lo, hi = dp["offsets"][e], dp["offsets"][e + 1]
        if hi > lo:
            assert rel_err(got_rows[lo:hi], ref_rows[lo:hi]) <= tol, "expert %d" % e
    if wl.d_ff_shared:
        sh_ref = oracle.expert_apply(dims, host["x"], weights_host(host), np.arange(T), np.full(T, E))
        assert rel_err(to_f64(st.y_perm[T * k:]), sh_ref) <= tol

    # ---- combine: same rows summed in float64, then compared at the output precision
    st.combine()
    assert st.status() == nat.MOE_OK
    yp = to_f64(st.y_perm)
    ref = np.zeros((T, wl.d_model))
    mag = np.zeros((T, wl.d_model))
    for t in range(T):
        for s in range(k):
            if ro[t, s] >= 0:
                ref[t] += yp[ro[t, s]]
                mag[t] += np.abs(yp[ro[t, s]])
        if wl.d_ff_shared:
            ref[t] += yp[T * k + t]
            mag[t] += np.abs(yp[T * k + t])
    got = to_f64(st.y)
    # one rounding to the output type plus the fp32 accumulation error
    out_ulp = 2.0 ** -8 if wl.dtype == "bf16" else 2.0 ** -23
    assert np.all(np.abs(got - ref) <= out_ulp * np.abs(ref) + 4e-7 * mag + 1e-30)

    # ---- balance statistics
    st.balance()
    bal = oracle.balance(dims, dp["counts"], r["pnorm"])
    # the forward pass computes them inside the dispatch kernels in the same
    # reduction order: identical bits
    out = nat.Outputs(st.cfg, cuda_device)
    nat.forward(st.cfg, inp, out, st.ws)
    assert torch.equal(out.f, st.f) and torch.equal(out.P, st.P) and torch.equal(out.loss, st.loss)
    # the forward pass runs the same kernels on the same operands in the same
    # order as the entry-point chain (its permute writes x_perm into the
    # workspace, its grouped FFN reads it from there): the same bits
    assert torch.equal(out.idx, st.idx) and torch.equal(out.y, st.y)
    assert abs(float(st.loss.item()) - bal["loss"]) <= TOL_LOSS * bal["loss"]
    np.testing.assert_allclose(st.f.cpu().numpy(), bal["f"], rtol=1e-6)
    np.testing.assert_allclose(st.P.cpu().numpy(), bal["P"], rtol=1e-4, atol=1e-7)


def test_permute_flags_bad_expert_id(cuda_device):
    wl = W("badid", T=64, d_model=64, E=4, d_ff=64, top_k=2)
    inp = syn.generate(wl, cuda_device, seed=0)
    st = Stage(wl, inp)
    st.idx.copy_(torch.tensor([[0, 1]] * 64, dtype=torch.int32))
    st.idx[5, 1] = 7                       # outside [0, E)
    st.gate.fill_(0.5)
    st.permute()
    assert st.status() == nat.MOE_ERR_DEVICE_BOUNDS
    assert int(st.row_of[5, 1].item()) == -1
    assert st.status() == nat.MOE_OK       # reading clears the word


def test_combine_flags_bad_row(cuda_device):
    wl = W("badrow", T=16, d_model=64, E=4, d_ff=64, top_k=2)
    inp = syn.generate(wl, cuda_device, seed=0)
    st = Stage(wl, inp)
    st.row_of.copy_(torch.arange(32, dtype=torch.int32).reshape(16, 2))
    st.row_of[3, 0] = 10_000
    st.combine()
    assert st.status() == nat.MOE_ERR_DEVICE_BOUNDS


def test_frozen_router_matches_the_per_call_split(cuda_device):
    """moe_router_freeze: a forward pass on a frozen workspace gives the same
    bits as one that splits W_r itself; new router weights (another tensor,
    or new values refrozen in place) are picked up; moe_workspace_init drops
    the freeze."""
    wl = W("frozen_router", T=300, d_model=256, E=16, d_ff=128, top_k=2, logit_skew="normal")
    dev = cuda_device
    inp = syn.generate(wl, dev, seed=5)
    cfg = nat.config_from_workload(wl)

    def run(ws, Wr):
        out = nat.Outputs(cfg, dev, want_logits=True)
        nat.forward(cfg, dict(inp, Wr=Wr), out, ws)
        torch.cuda.synchronize(dev)
        return out

    def same(a, b):
        return (torch.equal(a.y, b.y) and torch.equal(a.idx, b.idx) and torch.equal(a.gate, b.gate)
                and torch.equal(a.logits, b.logits))

    Wr = inp["Wr"]
    ref = run(nat.alloc_workspace(cfg, dev), Wr)
    ws = nat.alloc_workspace(cfg, dev)
    nat.moe_router_freeze(cfg, Wr, ws)
    assert same(run(ws, Wr), ref)
    assert same(run(ws, Wr), ref)                              # still frozen on the next call
    # other router weights: re-split, and the freeze is dropped
    Wr2 = Wr * 1.5
    ref2 = run(nat.alloc_workspace(cfg, dev), Wr2)
    assert same(run(ws, Wr2), ref2)
    assert same(run(ws, Wr), ref)                              # back to W_r: split again
    # new values in place need a new freeze
    nat.moe_router_freeze(cfg, Wr, ws)
    Wr.mul_(0.5)
    nat.moe_router_freeze(cfg, Wr, ws)
    ref3 = run(nat.alloc_workspace(cfg, dev), Wr)
    assert same(run(ws, Wr), ref3)
    nat.moe_workspace_init(ws)
    assert same(run(ws, Wr), ref3)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
