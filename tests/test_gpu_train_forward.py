"""GPU parity of the training forward (moe_forward_train through the C ABI):
the layer output equals moe_forward's bit for bit; the backward pass that
follows it on the same backward workspace uses the pre-activations the
forward saved and must give every gradient within the bf16 bound of the
oracle's backward (as test_gpu_backward.py) and within 4e-3 of the backward
that recomputes them; and a forward pass on the same forward workspace
between the two cancels the hand-over, so the backward recomputes from the
new inputs and matches the oracle for those.
"""
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat

from helpers import make_case, oracle_dims, rel_err, to_f64, weights_host
from test_gpu_backward import CASES, GRADS, TOL_GRAD

pytestmark = pytest.mark.gpu


def grads_close(a, b, tol):
    for name in GRADS:
        if a.get(name) is None:
            assert b.get(name) is None, name
            continue
        err = rel_err(to_f64(a[name]), to_f64(b[name]))
        assert err <= tol, (name, err)


def oracle_check(wl, host, dy, alpha, grads):
    ref = oracle.layer_backward(oracle_dims(wl), host["x"], host["Wr"], weights_host(host), to_f64(dy), alpha,
                                logit_bias=host["logit_bias"], sel_bias=host["sel_bias"])
    for name, rname in GRADS.items():
        if ref.get(rname) is None:
            assert grads.get(name) is None, name
            continue
        err = rel_err(to_f64(grads[name]), ref[rname])
        assert err <= TOL_GRAD, (name, err)


@pytest.mark.parametrize("wl,alpha", CASES, ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_training_forward_then_backward(wl, alpha, cuda_device):
    inp, host = make_case(wl, cuda_device, seed=2)
    cfg = nat.config_from_workload(wl)
    g = torch.Generator(device=cuda_device).manual_seed(9)
    dy = torch.randn((wl.T, wl.d_model), generator=g, device=cuda_device).to(torch.bfloat16)
    # the recomputing path
    out_a = nat.Outputs(cfg, want_logits=True)
    ws_a = nat.alloc_workspace(cfg)
    nat.forward(cfg, inp, out_a, ws_a)
    ga = nat.backward(cfg, inp, out_a, ws_a, dy, alpha)
    # the training forward and the backward on its workspace
    out_b = nat.Outputs(cfg, want_logits=True)
    ws_b = nat.alloc_workspace(cfg)
    bws = nat.alloc_backward_workspace(cfg, cuda_device)
    nat.forward_train(cfg, inp, out_b, ws_b, bws)
    gb = nat.backward(cfg, inp, out_b, ws_b, dy, alpha, ws=bws)
    torch.cuda.synchronize()
    for ws in (ws_a, ws_b):
        assert nat.moe_get_device_status(ws) == nat.MOE_OK, nat.last_error_detail()
    assert torch.equal(out_a.y, out_b.y)
    assert torch.equal(out_a.idx, out_b.idx)
    oracle_check(wl, host, dy, alpha, gb)
    grads_close(gb, ga, 4e-3)


def test_forward_between_cancels_the_hand_over(cuda_device):
    wl, alpha = CASES[0]
    inp1, _ = make_case(wl, cuda_device, seed=2)
    inp2, host2 = make_case(wl, cuda_device, seed=5)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, want_logits=True)
    ws = nat.alloc_workspace(cfg)
    bws = nat.alloc_backward_workspace(cfg, cuda_device)
    nat.forward_train(cfg, inp1, out, ws, bws)       # saves inp1's pre-activations in bws
    nat.forward(cfg, inp2, out, ws)                  # rewrites ws: the saved values no longer belong to it
    g = torch.Generator(device=cuda_device).manual_seed(3)
    dy = torch.randn((wl.T, wl.d_model), generator=g, device=cuda_device).to(torch.bfloat16)
    grads = nat.backward(cfg, inp2, out, ws, dy, alpha, ws=bws)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    oracle_check(wl, host2, dy, alpha, grads)


def test_hand_over_is_used_once(cuda_device):
    # a second backward on the same workspaces recomputes and agrees with the first
    wl, alpha = CASES[3]
    inp, host = make_case(wl, cuda_device, seed=4)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, want_logits=True)
    ws = nat.alloc_workspace(cfg)
    bws = nat.alloc_backward_workspace(cfg, cuda_device)
    nat.forward_train(cfg, inp, out, ws, bws)
    dy = torch.randn((wl.T, wl.d_model), device=cuda_device).to(torch.bfloat16)
    g1 = nat.backward(cfg, inp, out, ws, dy, alpha, ws=bws)
    g1 = {k: (v.clone() if v is not None else None) for k, v in g1.items()}
    g2 = nat.backward(cfg, inp, out, ws, dy, alpha, ws=bws)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    grads_close(g2, g1, 4e-3)
    oracle_check(wl, host, dy, alpha, g2)
