"""GPU parity of the block-scaled (MX) e4m3 expert path, through the C ABI,
against the oracle.

moe_quantize_rows_mx: codes and scale bytes equal byte for byte to the
  oracle's MX quantizer (both take the same fp32 decisions) on rows of many
  magnitudes, a zero row, a subnormal block and a row stride wider than the
  row;
moe_grouped_ffn_mx: every packed row (and every shared-expert row) against
  the oracle's MX expert on the same codes and scales, within the bf16 bound
  max|y - y_ref| / max|y_ref| <= 2e-2 per expert (H is rounded to bf16 and
  re-quantized on both sides; the GEMMs accumulate in fp32);
moe_forward_mx: routing as in the bf16 layer and y against the oracle's MX
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


@pytest.mark.parametrize("cols,ld,sld", [(32, 32, 16), (256, 256, 16), (2048, 2048, 64), (384, 400, 32)])
def test_quantize_rows_mx_matches_oracle(cols, ld, sld, cuda_device):
    g = torch.Generator(device=cuda_device)
    g.manual_seed(cols * 17 + ld)
    rows = 97
    x = torch.randn((rows, ld), generator=g, device=cuda_device)
    x *= torch.logspace(-6, 4, rows, device=cuda_device)[:, None]
    x[5] = 0.0
    x[7, 3] = -3e4                          # a negative block maximum
    x[9, :32] = 1e-39                       # a subnormal block: its exponent clamps at -127
    x = x.to(torch.bfloat16)
    codes = torch.full((rows, ld), 0xAB, dtype=torch.uint8, device=cuda_device)
    scales = torch.full((rows, sld), 0xCD, dtype=torch.uint8, device=cuda_device)
    nat.moe_quantize_rows_mx(x, codes, scales, cols=cols, ld_in=ld, ld_out=ld, ld_scale=sld)
    torch.cuda.synchronize(cuda_device)
    xh = x.float().cpu().numpy()[:, :cols]
    ref_c, ref_s = oracle.quantize_mx(xh)
    np.testing.assert_array_equal(codes[:, :cols].cpu().numpy(), ref_c)
    np.testing.assert_array_equal(scales[:, :cols // 32].cpu().numpy(), ref_s)
    assert bool((scales[:, cols // 32:] == 0xCD).all())           # bytes past each row's scales untouched
    if ld > cols:
        assert bool((codes[:, cols:] == 0xAB).all())


STAGE_CASES = [
    W("mx_stage_swiglu", T=640, d_model=256, E=12, d_ff=384, top_k=3, capacity_factor=0.9, logit_skew="normal"),
    W("mx_stage_gelu", T=500, d_model=384, E=8, d_ff=256, top_k=2, act="gelu"),
    W("mx_stage_shared", T=400, d_model=256, E=40, d_ff=128, top_k=6, score="sigmoid", sel_bias_std=0.1,
      d_ff_shared=256),
    W("mx_stage_wide", T=2048, d_model=1024, E=16, d_ff=768, top_k=4, logit_skew="zipf"),
]


@pytest.mark.parametrize("wl", STAGE_CASES, ids=lambda w: w.name)
def test_grouped_ffn_mx_rows(wl, cuda_device):
    dev = cuda_device
    inp = syn.generate(wl, dev, 17, weights=False)
    host = to_host(inp)
    enforce_margin(wl, inp, host, 17)
    cfg = nat.config_from_workload(wl)
    sld = nat.mx_sld(cfg)
    w = syn.generate_mx_experts(wl, sld, dev, seed=17)
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
    xs = torch.zeros((T, sld), dtype=torch.uint8, device=dev)
    nat.moe_quantize_rows_mx(inp["x"], x8, xs)
    torch.cuda.synchronize(dev)
    nrows = int(offsets[-1].item())
    rt = row_token[:nrows].long()
    x8_perm = torch.zeros((T * k, d), dtype=torch.uint8, device=dev)
    x8_perm[:nrows] = x8[rt]
    xs_perm = torch.zeros((T * k, sld), dtype=torch.uint8, device=dev)
    xs_perm[:nrows] = xs[rt]
    y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    mws = torch.empty(nat.grouped_ffn_mx_workspace_size(cfg, sld), dtype=torch.uint8, device=dev)
    mws[:256].zero_()
    nat.moe_grouped_ffn_mx(cfg, x8_perm, xs_perm, offsets, row_gate, w, sld, w.get("b1"), w.get("b2"), x8, xs,
                           y_perm, mws)
    torch.cuda.synchronize(dev)
    assert nat.moe_get_device_status(mws) == nat.MOE_OK, nat.last_error_detail()

    dims = oracle_dims(wl)
    x8h, xsh = oracle.quantize_mx(oracle.bf16_bits_to_f64(host["x"]).astype(np.float32))
    assert np.array_equal(x8.cpu().numpy(), x8h) and np.array_equal(xs[:, :d // 32].cpu().numpy(), xsh)
    wh = {}
    for name, v in w.items():
        if v is None:
            continue
        a = v.cpu().numpy()
        if name.endswith("_scale"):
            K = (d if name[:-6] in ("W1", "Wu", "Wsg", "Wsu") else
                 (wl.d_ff_shared if name.startswith("Wsd") else wl.d_ff))
            a = np.ascontiguousarray(a[..., :K // 32])
        wh[name] = a
    off = offsets.cpu().numpy()
    row_expert = np.repeat(np.arange(E), np.diff(off)).astype(np.int32)
    ref = oracle.expert_apply_mx(dims, x8h, xsh, wh, row_token[:nrows].cpu().numpy(), row_expert,
                                 row_gate[:nrows].double().cpu().numpy())
    got = to_f64(y_perm[:nrows])
    for e in range(E):
        if off[e + 1] > off[e]:
            err = rel_err(got[off[e]:off[e + 1]], ref[off[e]:off[e + 1]])
            assert err <= TOL_BF16, "expert %d: %.3e" % (e, err)
    if wl.d_ff_shared:
        sh = oracle.expert_apply_mx(dims, x8h, xsh, wh, np.arange(T, dtype=np.int32), np.full(T, E, np.int32))
        assert rel_err(to_f64(y_perm[T * k:]), sh) <= TOL_BF16


def mx_host_weights(wl, w):
    """The device MX weights as host arrays, scale rows cut to their K / 32 bytes."""
    wh = {}
    for name, v in w.items():
        if v is None:
            continue
        a = v.cpu().numpy()
        if name.endswith("_scale"):
            base = name[:-6]
            K = (wl.d_model if base in ("W1", "Wu", "Wsg", "Wsu") else
                 (wl.d_ff_shared if base == "Wsd" else wl.d_ff))
            a = np.ascontiguousarray(a[..., :K // 32])
        wh[name] = a
    return wh


def check_mx_forward(wl, dev, seed=0, n_sample=None):
    """moe_forward_mx: routing as in the bf16 layer, and y against the oracle's
    MX layer on the oracle's own MX codes of x (every token, or sampled tokens
    covering every expert with a kept row)."""
    inp = syn.generate(wl, dev, seed, weights=False)
    host = to_host(inp)
    if wl.T > 0 and wl.top_k < wl.E:
        enforce_margin(wl, inp, host, seed)
    cfg = nat.config_from_workload(wl)
    sld = nat.mx_sld(cfg)
    w = syn.generate_mx_experts(wl, sld, dev, seed=seed)
    out = nat.Outputs(cfg, dev)
    ws = nat.alloc_workspace(cfg, dev)
    mws = nat.alloc_mx_workspace(cfg, sld, dev)
    nat.forward_mx(cfg, inp, w, sld, out, ws, mws)
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
    x8h, xsh = oracle.quantize_mx(oracle.bf16_bits_to_f64(host["x"]).astype(np.float32))
    y_ref = oracle.layer_tokens_mx(dims, x8h, xsh, mx_host_weights(wl, w), r["idx"], r["gate"], dp["row_of"],
                                   tokens)
    err = rel_err(to_f64(out.y)[tokens], y_ref)
    assert err <= TOL_BF16, "max|y-y_ref|/max|y_ref| = %.3e" % err
    return err


FORWARD_CASES = [
    W("mx_switch", T=600, d_model=256, E=16, d_ff=384, top_k=1, act="gelu", renorm=0, capacity_factor=1.25,
      logit_skew="normal"),
    W("mx_mixtral", T=520, d_model=384, E=8, d_ff=512, top_k=2),
    W("mx_qwen", T=700, d_model=256, E=32, d_ff=256, top_k=8, logit_skew="zipf"),
    W("mx_deepseek", T=333, d_model=512, E=64, d_ff=256, top_k=8, score="sigmoid", d_ff_shared=384,
      sel_bias_std=0.1),
]


@pytest.mark.parametrize("wl", FORWARD_CASES, ids=lambda w: w.name)
def test_forward_mx_small(wl, cuda_device):
    check_mx_forward(wl, cuda_device, seed=3)


def test_forward_mx_qwen3_full_size(cuda_device):
    err = check_mx_forward(syn.WORKLOADS["qwen3_moe"], cuda_device, seed=0, n_sample=32)
    print("qwen3_moe mx: max rel err %.3e" % err)


@pytest.mark.parametrize("T", [0, 1, 33])
def test_forward_mx_tiny_T(T, cuda_device):
    wl = W("mx_tiny", T=T, d_model=128, E=8, d_ff=128, top_k=2, d_ff_shared=128)
    if T == 0:
        cfg = nat.config_from_workload(wl)
        inp = syn.generate(wl.replace(T=1), cuda_device, 1, weights=False)
        sld = nat.mx_sld(cfg)
        w = syn.generate_mx_experts(wl, sld, cuda_device, seed=1)
        out = nat.Outputs(cfg, cuda_device)
        ws = nat.alloc_workspace(cfg, cuda_device)
        nat.forward_mx(cfg, inp, w, sld, out, ws, nat.alloc_mx_workspace(cfg, sld, cuda_device))
        torch.cuda.synchronize(cuda_device)
        assert not out.counts.any().item()
        return
    check_mx_forward(wl, cuda_device, seed=1)
