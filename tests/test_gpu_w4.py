"""GPU parity of the INT4 weight-only expert path, through the C ABI, against
the oracle.

moe_grouped_ffn_w4: every packed row (and every shared-expert row) against
  the oracle's INT4 expert on the same bf16 rows and packed weights, within
  the bf16 bound max|y - y_ref| / max|y_ref| <= 2e-2 per expert (weights
  decode to the same bf16 values on both sides; H is held in bf16 on the GPU
  and exact in the oracle, as for bf16 experts);
moe_forward_w4: routing as in the bf16 layer and y against the oracle's INT4
  layer -- every token on small cases (Switch-, Mixtral-, Qwen3- and
  DeepSeek-like, GELU and SwiGLU, capacity drops, a shared expert), sampled
  tokens covering every expert on the full-size Qwen3 workload, T in
  {0, 1, 33} -- within the same bound.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import (TOL_BF16, check_routing, enforce_margin, oracle_dims, rel_err, sample_tokens, to_f64,
                     to_host)

pytestmark = pytest.mark.gpu

W = syn.Workload


def w4_host_weights(wl, w):
    """Device INT4 weights as host arrays: codes as they are, scale rows cut
    to their K / 128 bf16 values (uint16 bits)."""
    wh = {}
    for name, v in w.items():
        if v is None:
            continue
        a = v.cpu().numpy()
        if name.endswith("_scale"):
            base = name[:-6]
            K = (wl.d_model if base in ("W1", "Wu", "Wsg", "Wsu") else
                 (wl.d_ff_shared if base == "Wsd" else wl.d_ff))
            a = np.ascontiguousarray(a[..., :2 * (K // 128)]).view(np.uint16)
        wh[name] = a
    return wh


STAGE_CASES = [
    W("w4_stage_swiglu", T=640, d_model=256, E=12, d_ff=384, top_k=3, capacity_factor=0.9, logit_skew="normal"),
    W("w4_stage_gelu", T=500, d_model=384, E=8, d_ff=256, top_k=2, act="gelu"),
    W("w4_stage_shared", T=400, d_model=256, E=40, d_ff=128, top_k=6, score="sigmoid", sel_bias_std=0.1,
      d_ff_shared=256),
    W("w4_stage_wide", T=2048, d_model=1024, E=16, d_ff=768, top_k=4, logit_skew="zipf"),
]


@pytest.mark.parametrize("wl", STAGE_CASES, ids=lambda w: w.name)
def test_grouped_ffn_w4_rows(wl, cuda_device):
    dev = cuda_device
    inp = syn.generate(wl, dev, 19, weights=False)
    host = to_host(inp)
    enforce_margin(wl, inp, host, 19)
    cfg = nat.config_from_workload(wl)
    sld = nat.w4_sld(cfg)
    w = syn.generate_w4_experts(wl, sld, dev, seed=19)
    T, k, E, d = wl.T, wl.top_k, wl.E, wl.d_model
    ws = nat.alloc_workspace(cfg, dev)
    idx = torch.empty((T, k), dtype=torch.int32, device=dev)
    gate = torch.empty((T, k), dtype=torch.float32, device=dev)
    psum = torch.empty((nat.router_blocks(cfg), E), dtype=torch.float32, device=dev)
    nat.moe_router_topk(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"], idx, gate, None, psum, ws)
    counts = torch.empty(E, dtype=torch.int32, device=dev)
    kept = torch.empty(E, dtype=torch.int32, device=dev)
    offsets = torch.empty(E + 1, dtype=torch.int32, device=dev)
    row_of = torch.empty((T, k), dtype=torch.int32, device=dev)
    row_token = torch.zeros(T * k, dtype=torch.int32, device=dev)
    row_gate = torch.zeros(T * k, dtype=torch.float32, device=dev)
    x_perm = torch.zeros((T * k, d), dtype=torch.bfloat16, device=dev)
    nat.moe_permute(cfg, inp["x"], idx, gate, counts, kept, offsets, row_of, row_token, row_gate, x_perm, None, ws)
    y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    nat.moe_grouped_ffn_w4(cfg, x_perm, offsets, row_gate, w, sld, w.get("b1"), w.get("b2"), inp["x"], y_perm, ws)
    torch.cuda.synchronize(dev)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK, nat.last_error_detail()

    dims = oracle_dims(wl)
    wh = w4_host_weights(wl, w)
    nrows = int(offsets[-1].item())
    off = offsets.cpu().numpy()
    row_expert = np.repeat(np.arange(E), np.diff(off)).astype(np.int32)
    ref = oracle.expert_apply_w4(dims, host["x"], wh, row_token[:nrows].cpu().numpy(), row_expert,
                                 row_gate[:nrows].double().cpu().numpy())
    got = to_f64(y_perm[:nrows])
    for e in range(E):
        if off[e + 1] > off[e]:
            err = rel_err(got[off[e]:off[e + 1]], ref[off[e]:off[e + 1]])
            assert err <= TOL_BF16, "expert %d: %.3e" % (e, err)
    if wl.d_ff_shared:
        sh = oracle.expert_apply_w4(dims, host["x"], wh, np.arange(T, dtype=np.int32), np.full(T, E, np.int32))
        assert rel_err(to_f64(y_perm[T * k:]), sh) <= TOL_BF16


def check_w4_forward(wl, dev, seed=0, n_sample=None):
    inp = syn.generate(wl, dev, seed, weights=False)
    host = to_host(inp)
    if wl.T > 0 and wl.top_k < wl.E:
        enforce_margin(wl, inp, host, seed)
    cfg = nat.config_from_workload(wl)
    sld = nat.w4_sld(cfg)
    w = syn.generate_w4_experts(wl, sld, dev, seed=seed)
    out = nat.Outputs(cfg, dev)
    ws = nat.alloc_workspace(cfg, dev)
    nat.forward_w4(cfg, inp, w, sld, out, ws)
    torch.cuda.synchronize(dev)
    status = nat.moe_get_device_status(ws)
    assert status == nat.MOE_OK, nat.status_string(status)
    dims = oracle_dims(wl)
    r = oracle.route(dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"])
    dp = oracle.dispatch(dims, r["idx"])
    check_routing(out.idx.cpu().numpy(), out.gate.cpu().numpy(), r)
    np.testing.assert_array_equal(out.counts.cpu().numpy(), dp["counts"])
    if n_sample is None:
        tokens = np.arange(wl.T, dtype=np.int32)
    else:
        tokens = sample_tokens(r["idx"], dp["row_of"], wl.E, n_sample, seed, wl.T)
    y_ref = oracle.layer_tokens_w4(dims, host["x"], w4_host_weights(wl, w), r["idx"], r["gate"], dp["row_of"],
                                   tokens)
    err = rel_err(to_f64(out.y)[tokens], y_ref)
    assert err <= TOL_BF16, "max|y-y_ref|/max|y_ref| = %.3e" % err
    return err


FORWARD_CASES = [
    W("w4_switch", T=600, d_model=256, E=16, d_ff=384, top_k=1, act="gelu", renorm=0, capacity_factor=1.25,
      logit_skew="normal"),
    W("w4_mixtral", T=520, d_model=384, E=8, d_ff=512, top_k=2),
    W("w4_qwen", T=700, d_model=256, E=32, d_ff=256, top_k=8, logit_skew="zipf"),
    W("w4_deepseek", T=333, d_model=512, E=64, d_ff=256, top_k=8, score="sigmoid", d_ff_shared=384,
      sel_bias_std=0.1),
]


@pytest.mark.parametrize("wl", FORWARD_CASES, ids=lambda w: w.name)
def test_forward_w4_small(wl, cuda_device):
    check_w4_forward(wl, cuda_device, seed=4)


def test_forward_w4_qwen3_full_size(cuda_device):
    err = check_w4_forward(syn.WORKLOADS["qwen3_moe"], cuda_device, seed=0, n_sample=32)
    print("qwen3_moe w4: max rel err %.3e" % err)


@pytest.mark.parametrize("T", [0, 1, 33])
def test_forward_w4_tiny_T(T, cuda_device):
    wl = W("w4_tiny", T=T, d_model=128, E=8, d_ff=128, top_k=2, d_ff_shared=128)
    if T == 0:
        cfg = nat.config_from_workload(wl)
        inp = syn.generate(wl.replace(T=1), cuda_device, 1, weights=False)
        sld = nat.w4_sld(cfg)
        w = syn.generate_w4_experts(wl, sld, cuda_device, seed=1)
        out = nat.Outputs(cfg, cuda_device)
        nat.forward_w4(cfg, inp, w, sld, out, nat.alloc_workspace(cfg, cuda_device))
        torch.cuda.synchronize(cuda_device)
        assert not out.counts.any().item()
        return
    check_w4_forward(wl, cuda_device, seed=1)
