"""GPU parity of the FP8 (e4m3) expert path, through the C ABI, against the
oracle.

moe_quantize_rows_e4m3: codes and scales byte for byte equal to the oracle's
  quantizer (both take the same fp32 decisions) on rows of several
  magnitudes, a zero row and a row stride wider than the row;
moe_grouped_ffn_fp8: every packed row against the oracle's FP8 expert on the
  same e4m3 inputs;
moe_forward_fp8: routing as in the bf16 layer and y against the oracle's FP8
  layer -- every token on small cases (ragged widths that leave partial K and
  N tiles included), on the full-size workloads sampled tokens that cover
  every expert with a kept row -- within the bf16 bound
  max|y - y_ref| / max|y_ref| <= 2e-2.
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


def make_fp8_case(wl, dev, seed):
    inp = syn.generate(wl, dev, seed, weights=False)
    host = to_host(inp)
    if wl.T > 0 and wl.top_k < wl.E:
        enforce_margin(wl, inp, host, seed)
    w8 = syn.generate_fp8_experts(wl, dev, seed)
    inp["b1"], inp["b2"] = w8.get("b1"), w8.get("b2")
    w8h = {k: v.cpu().numpy() for k, v in w8.items() if v is not None}
    return inp, host, w8, w8h


def host_x8(host):
    return oracle.quantize_rows(oracle.bf16_bits_to_f64(host["x"]).astype(np.float32))


@pytest.mark.parametrize("cols,ld", [(8, 8), (200, 200), (2048, 2048), (136, 152)])
def test_quantize_rows_matches_oracle(cols, ld, cuda_device):
    g = torch.Generator(device=cuda_device)
    g.manual_seed(cols * 31 + ld)
    rows = 97
    x = torch.randn((rows, ld), generator=g, device=cuda_device)
    x *= torch.logspace(-4, 3, rows, device=cuda_device)[:, None]
    x[5] = 0.0
    x[7, 3] = -1e4                          # a negative row maximum
    x = x.to(torch.bfloat16)
    codes = torch.full((rows, ld), 0xAB, dtype=torch.uint8, device=cuda_device)
    scale = torch.empty(rows, dtype=torch.float32, device=cuda_device)
    nat.moe_quantize_rows_e4m3(x, codes, scale, cols=cols, ld_in=ld, ld_out=ld)
    torch.cuda.synchronize(cuda_device)
    xh = x.float().cpu().numpy()[:, :cols]
    ref_c, ref_s = oracle.quantize_rows(xh)
    np.testing.assert_array_equal(codes[:, :cols].cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scale.cpu().numpy(), ref_s)
    if ld > cols:                           # bytes past each row are not written
        assert bool((codes[:, cols:] == 0xAB).all())


STAGE_CASES = [
    W("f8_stage_swiglu", T=640, d_model=256, E=12, d_ff=320, top_k=3, capacity_factor=0.9, logit_skew="normal"),
    W("f8_stage_gelu", T=500, d_model=192, E=8, d_ff=256, top_k=2, act="gelu"),
    W("f8_stage_shared", T=400, d_model=384, E=40, d_ff=128, top_k=6, score="sigmoid", sel_bias_std=0.1,
      d_ff_shared=256),
]


@pytest.mark.parametrize("wl", STAGE_CASES, ids=lambda w: w.name)
def test_grouped_ffn_fp8_rows(wl, cuda_device):
    dev = cuda_device
    inp, host, w8, w8h = make_fp8_case(wl, dev, seed=13)
    cfg = nat.config_from_workload(wl)
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
    nat.moe_permute(cfg, inp["x"], idx, gate, counts, kept, offsets, row_of, row_token, row_gate, None, None, ws)
    x8 = torch.empty((T, d), dtype=torch.uint8, device=dev)
    xs = torch.empty(T, dtype=torch.float32, device=dev)
    nat.moe_quantize_rows_e4m3(inp["x"], x8, xs)
    torch.cuda.synchronize(dev)
    nrows = int(offsets[-1].item())
    rt = row_token[:nrows].long()
    x8_perm = torch.zeros((T * k, d), dtype=torch.uint8, device=dev)
    x8_perm[:nrows] = x8[rt]
    xps = torch.zeros(T * k, dtype=torch.float32, device=dev)
    xps[:nrows] = xs[rt]
    y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    nat.moe_grouped_ffn_fp8(cfg, x8_perm, xps, offsets, row_gate, w8, inp["b1"], inp["b2"], x8, xs, y_perm, ws)
    torch.cuda.synchronize(dev)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK

    dims = oracle_dims(wl)
    x8h, xsh = host_x8(host)
    assert np.array_equal(x8.cpu().numpy(), x8h) and np.array_equal(xs.cpu().numpy(), xsh)
    off = offsets.cpu().numpy()
    row_expert = np.repeat(np.arange(E), np.diff(off)).astype(np.int32)
    ref = oracle.expert_apply_fp8(dims, x8h, xsh, w8h, row_token[:nrows].cpu().numpy(), row_expert,
                                  row_gate[:nrows].double().cpu().numpy())
    got = to_f64(y_perm[:nrows])
    for e in range(E):
        if off[e + 1] > off[e]:
            err = rel_err(got[off[e]:off[e + 1]], ref[off[e]:off[e + 1]])
            assert err <= TOL_BF16, "expert %d: %.3e" % (e, err)
    if wl.d_ff_shared:
        sh = oracle.expert_apply_fp8(dims, x8h, xsh, w8h, np.arange(T, dtype=np.int32), np.full(T, E, np.int32))
        assert rel_err(to_f64(y_perm[T * k:]), sh) <= TOL_BF16


def check_fp8_forward(wl, dev, seed=0, n_sample=None):
    inp, host, w8, w8h = make_fp8_case(wl, dev, seed)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, dev)
    ws = nat.alloc_workspace(cfg, dev)
    nat.forward_fp8(cfg, inp, w8, out, ws)
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
    x8h, xsh = host_x8(host)
    y_ref = oracle.layer_tokens_fp8(dims, x8h, xsh, w8h, r["idx"], r["gate"], dp["row_of"], tokens)
    err = rel_err(to_f64(out.y)[tokens], y_ref)
    assert err <= TOL_BF16, "max|y-y_ref|/max|y_ref| = %.3e" % err
    return err, out


SMALL = [
    W("f8_switch", T=600, d_model=256, E=16, d_ff=384, top_k=1, act="gelu", renorm=0, capacity_factor=1.25,
      logit_skew="normal"),
    W("f8_mixtral", T=520, d_model=384, E=8, d_ff=448, top_k=2),
    W("f8_qwen", T=700, d_model=256, E=32, d_ff=192, top_k=8, logit_skew="zipf"),
    W("f8_deepseek", T=333, d_model=512, E=64, d_ff=256, top_k=8, score="sigmoid", d_ff_shared=384,
      sel_bias_std=0.1),
    W("f8_ragged", T=301, d_model=208, E=5, d_ff=144, top_k=2, act="gelu", d_ff_shared=80),
]


@pytest.mark.parametrize("wl", SMALL, ids=lambda w: w.name)
def test_forward_fp8_small(wl, cuda_device):
    check_fp8_forward(wl, cuda_device, seed=2)


@pytest.mark.parametrize("name", ["switch_top1", "mixtral", "qwen3_moe", "deepseek_v3"])
def test_forward_fp8_full_size(name, cuda_device):
    wl = syn.WORKLOADS[name]
    err, _ = check_fp8_forward(wl, cuda_device, seed=0, n_sample=32)
    print("%s fp8: max rel err %.3e" % (name, err))


@pytest.mark.parametrize("T", [0, 1, 33])
def test_forward_fp8_tiny_T(T, cuda_device):
    wl = W("f8_tiny", T=T, d_model=128, E=8, d_ff=128, top_k=2, d_ff_shared=64)
    if T == 0:
        inp, _, w8, _ = make_fp8_case(wl, cuda_device, seed=1)
        cfg = nat.config_from_workload(wl)
        out = nat.Outputs(cfg, cuda_device)
        ws = nat.alloc_workspace(cfg, cuda_device)
        nat.forward_fp8(cfg, inp, w8, out, ws)
        torch.cuda.synchronize(cuda_device)
        assert not out.counts.any().item()
        return
    check_fp8_forward(wl, cuda_device, seed=1)


def test_fp8_rejects_unsupported(cuda_device):
    wl = W("f8_bad", T=16, d_model=72, E=4, d_ff=64, top_k=2)     # d_model not a multiple of 16
    inp, _, w8, _ = make_fp8_case(W("f8_ok", T=16, d_model=80, E=4, d_ff=64, top_k=2), cuda_device, seed=0)
    cfg = nat.config_from_workload(wl)
    out = nat.Outputs(cfg, cuda_device)
    ws = nat.alloc_workspace(cfg, cuda_device)
    with pytest.raises(nat.MoEError) as ei:
        nat.forward_fp8(cfg, inp, w8, out, ws)
    assert ei.value.status == nat.MOE_ERR_UNSUPPORTED
