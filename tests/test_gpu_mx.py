"""GPU parity of the block-scaled (MX) e4m3 expert path, through the C ABI,
against the oracle.

moe_quantize_rows_mx: codes and scale bytes equal byte for byte to the
  oracle's MX quantizer (both take the same fp32 decisions) on rows of many
  magnitudes, a zero row, a subnormal block and a row stride wider than the
  row;
moe_grouped_ffn_mx: every packed row (and every shared-expert row) against
  the oracle's MX expert on the same codes and scales, within the bf16 bound
  max|y - y_ref| / max|y_ref| <= 2e-2 per expert (H is rounded to bf16 and
  re-quantized on both sides; the GEMMs accumulate in fp32).
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import TOL_BF16, enforce_margin, oracle_dims, rel_err, to_f64, to_host

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
