"""GPU parity of the auxiliary-loss-free bias update and the routing-health
statistics (entropy of the mean routing distribution, max/min utilisation
ratio, largest share) against the oracle, through the C ABI."""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import make_case, oracle_dims

pytestmark = pytest.mark.gpu


def test_bias_update_matches_oracle(cuda_device):
    T, k, E = 1000, 4, 64
    cfg = nat.make_config(T, 64, E, 64, k)
    rng = np.random.default_rng(3)
    counts = rng.integers(0, 2 * T * k // E, E).astype(np.int32)
    bias = rng.normal(0, 0.1, E).astype(np.float32)
    gamma = float(np.float32(0.001))
    c_d = torch.from_numpy(counts).to(cuda_device)
    b_d = torch.from_numpy(bias).to(cuda_device)
    nat.moe_bias_update(cfg, c_d, b_d, gamma)
    dims = oracle.make_dims(T, 64, E, 64, k, x_dtype="bf16")
    np.testing.assert_array_equal(b_d.cpu().numpy(), oracle.bias_update(dims, counts, bias, gamma))


def test_bias_update_exact_target_keeps_bias(cuda_device):
    T, k, E = 64, 2, 8                  # target 16
    cfg = nat.make_config(T, 64, E, 64, k)
    counts = torch.tensor([16, 17, 15, 16, 0, 32, 16, 16], dtype=torch.int32, device=cuda_device)
    b = torch.zeros(E, dtype=torch.float32, device=cuda_device)
    nat.moe_bias_update(cfg, counts, b, 0.5)
    assert b.cpu().tolist() == [0.0, -0.5, 0.5, 0.0, 0.5, -0.5, 0.0, 0.0]


def test_routing_health_matches_oracle(cuda_device):
    wl = syn.WORKLOADS["qwen3_moe"].replace(name="health", T=2048)
    inp, host = make_case(wl, cuda_device, seed=4)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, cuda_device)
    ws = nat.alloc_workspace(cfg, cuda_device)
    nat.forward(cfg, inp, out, ws)
    health = torch.empty(3, dtype=torch.float64, device=cuda_device)
    nat.moe_routing_health(cfg, out.counts, out.P, health)
    dims = oracle_dims(wl)
    r = oracle.route(dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"])
    counts = oracle.dispatch(dims, r["idx"])["counts"]
    ref = oracle.routing_health(dims, counts, oracle.balance(dims, counts, r["pnorm"])["P"])
    got = health.cpu().numpy()
    assert abs(got[0] - ref["entropy"]) <= 1e-5 * ref["entropy"]
    assert got[1] == ref["ratio"] and got[2] == ref["max_share"]


def test_bias_steps_on_device_balance_a_skewed_router(cuda_device):
    # forward -> counts -> bias update, repeated on the device: the hot
    # expert's load falls
    wl = syn.Workload("bias_loop", T=512, d_model=64, E=16, d_ff=64, top_k=2, score="sigmoid",
                      sel_bias_std=0.0)
    inp = syn.generate(wl, cuda_device, seed=9)
    inp["logit_bias"] = torch.tensor([2.0, 1.5] + [0.0] * 14, device=cuda_device)
    inp["sel_bias"] = torch.zeros(16, device=cuda_device)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, cuda_device)
    ws = nat.alloc_workspace(cfg, cuda_device)
    loads = []
    for _ in range(60):
        nat.forward(cfg, inp, out, ws)
        loads.append(int(out.counts.max().item()))
        nat.moe_bias_update(cfg, out.counts, inp["sel_bias"], 0.02)
    assert loads[-1] < loads[0] * 0.75
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
