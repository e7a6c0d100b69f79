"""GPU parity of the backward pass (moe_backward through the C ABI) against
the oracle's backward (fp64), which finite differences pin
(test_oracle_backward_pins.py).

After moe_forward on seeded inputs (selection margin enforced), moe_backward
with a seeded upstream gradient dy and an aux-loss weight alpha must give
every gradient within max|g - g_ref| / max|g_ref| <= 2e-2: the bound of the
bf16 layer, since the contractions run on bf16 operands (dy scaled by the
gates, the recomputed pre-activations and their gradients, the router's
logit gradient) with fp32 accumulation.  Cases cover renormalised softmax
gates with SwiGLU experts, full-softmax gates with GELU experts, biases and
capacity drops, sigmoid gates with a selection bias and a shared expert,
group sizes across tile boundaries, and an expert that keeps no row (its
weight gradient must be exactly zero).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import make_case, oracle_dims, rel_err, to_f64, weights_host

pytestmark = pytest.mark.gpu

W = syn.Workload
TOL_GRAD = 2e-2

CASES = [
    (W("bwd_swiglu", T=384, d_model=256, E=8, d_ff=192, top_k=2, logit_skew="zipf"), 0.5),
    (W("bwd_gelu_cap", T=320, d_model=128, E=4, d_ff=256, top_k=2, act="gelu", renorm=0, capacity_factor=0.7,
       logit_skew="normal"), 0.2),
    (W("bwd_sigmoid_shared", T=256, d_model=192, E=16, d_ff=128, top_k=4, score="sigmoid", sel_bias_std=0.1,
       d_ff_shared=128), 1.0),
    (W("bwd_qwen_like", T=1024, d_model=512, E=32, d_ff=256, top_k=8, logit_skew="zipf"), 0.01),
]

GRADS = {"dx": "dx", "dWr": "dWr", "dlogit_bias": "dbeta", "dW1": "dW1", "dWu": "dWu", "dW2": "dW2", "db1": "db1",
         "db2": "db2", "dWsg": "dWsg", "dWsu": "dWsu", "dWsd": "dWsd"}


@pytest.mark.parametrize("wl,alpha", CASES, ids=lambda v: v.name if hasattr(v, "name") else str(v))
def test_backward_against_oracle(wl, alpha, cuda_device):
    inp, host = make_case(wl, cuda_device, seed=2)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, want_logits=True)
    ws = nat.alloc_workspace(cfg)
    nat.forward(cfg, inp, out, ws)
    g = torch.Generator(device=cuda_device).manual_seed(9)
    dy = torch.randn((wl.T, wl.d_model), generator=g, device=cuda_device).to(torch.bfloat16)
    grads = nat.backward(cfg, inp, out, ws, dy, alpha)
    status = nat.moe_get_device_status(ws)
    assert status == nat.MOE_OK, nat.last_error_detail()
    dims = oracle_dims(wl)
    ref = oracle.layer_backward(dims, host["x"], host["Wr"], weights_host(host), to_f64(dy), alpha,
                                logit_bias=host["logit_bias"], sel_bias=host["sel_bias"])
    report = {}
    for name, rname in GRADS.items():
        got = grads.get(name)
        if ref.get(rname) is None:
            assert got is None, name
            continue
        if name == "dlogit_bias" and host["logit_bias"] is None:
            # no logit offset in the layer: its gradient is still defined (d ell / d beta)
            pass
        err = rel_err(to_f64(got), ref[rname])
        report[name] = err
        assert err <= TOL_GRAD, (name, err)
    print(wl.name, {k: "%.2e" % v for k, v in report.items()})


def test_backward_expert_without_rows_gets_zero(cuda_device):
    # a logit offset of -30 keeps expert 3 out of every top-2
    wl = W("bwd_idle_expert", T=256, d_model=128, E=4, d_ff=128, top_k=2)
    inp, host = make_case(wl, cuda_device, seed=8)
    lb = torch.tensor([0.0, 0.0, 0.0, -30.0], device=cuda_device)
    inp["logit_bias"] = lb
    host["logit_bias"] = lb.cpu().numpy()
    from helpers import enforce_margin
    enforce_margin(wl, inp, host, seed=8)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, want_logits=True)
    ws = nat.alloc_workspace(cfg)
    nat.forward(cfg, inp, out, ws)
    assert int(out.counts[3].item()) == 0
    dy = torch.randn((wl.T, wl.d_model), device=cuda_device).to(torch.bfloat16)
    grads = nat.backward(cfg, inp, out, ws, dy, 0.1)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    for name in ("dW1", "dWu", "dW2"):
        assert torch.count_nonzero(grads[name][3]).item() == 0
        assert torch.count_nonzero(grads[name][0]).item() > 0


def test_backward_refuses_unsupported(cuda_device):
    cfg = nat.make_config(64, 96, 4, 128, 2)          # d_model not a multiple of 64
    assert nat.lib().moe_backward_workspace_size(cfg) == 0
    cfg = nat.make_config(64, 128, 4, 128, 2, dtype="f32")
    assert nat.lib().moe_backward_workspace_size(cfg) == 0
