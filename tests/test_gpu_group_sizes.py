"""The grouped expert FFN entry point on hand-made group sizes, against the
oracle expert applied row by row.

The sizes straddle every tile boundary of the tensor-core path: empty groups,
groups of 1..128 rows (the 1-CTA kernel's 128-row tiles), 256-row blocks
(CTA-pair tiles) with and without a last block of 1..128 rows, and a last
block of more than 128 rows (a pair tile with padding).  d_ff and d_model are
not multiples of the weight tiles, so partial weight tiles are covered too;
one case adds a shared expert.  The same sizes also go through the e4m3
(FP8) grouped FFN.
"""
import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import TOL_BF16, oracle_dims, rel_err, to_f64, to_host, weights_host

pytestmark = pytest.mark.gpu

SIZES = [0, 1, 31, 32, 33, 63, 64, 65, 127, 128, 129, 200, 255, 256, 257, 383, 384, 385, 513, 640]

CASES = [
    syn.Workload("sizes_swiglu", T=1000, d_model=384, E=len(SIZES), d_ff=320, top_k=4),
    syn.Workload("sizes_gelu", T=1000, d_model=192, E=len(SIZES), d_ff=320, top_k=4, act="gelu", renorm=0),
    syn.Workload("sizes_shared", T=1000, d_model=256, E=len(SIZES), d_ff=192, top_k=4, d_ff_shared=320),
]


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_group_sizes(wl, cuda_device):
    dev = cuda_device
    inp = syn.generate(wl, dev, seed=21)
    host = to_host(inp)
    cfg = nat.config_from_workload(wl)
    T, k, E, d = wl.T, wl.top_k, wl.E, wl.d_model
    rng = np.random.default_rng(5)
    sizes = np.array(SIZES, np.int64)
    rng.shuffle(sizes)                     # group order independent of size
    nrows = int(sizes.sum())
    assert nrows <= T * k
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(sizes)
    row_token = rng.integers(0, T, T * k).astype(np.int32)
    row_gate = rng.uniform(0.05, 1.0, T * k).astype(np.float32)
    x_perm = inp["x"][torch.from_numpy(row_token.astype(np.int64)).to(dev)].contiguous()
    y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=inp["x"].dtype, device=dev)
    ws = nat.alloc_workspace(cfg, dev)
    nat.moe_grouped_ffn(cfg, x_perm, torch.from_numpy(offsets).to(dev), torch.from_numpy(row_gate).to(dev),
                        inp["W1"], inp["b1"], inp["Wu"], inp["W2"], inp["b2"], inp["x"], inp["Wsg"], inp["Wsu"],
                        inp["Wsd"], y_perm, ws)
    torch.cuda.synchronize(dev)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK

    dims = oracle_dims(wl)
    row_expert = np.repeat(np.arange(E), sizes).astype(np.int32)
    ref = oracle.expert_apply(dims, host["x"], weights_host(host), row_token[:nrows], row_expert,
                              row_gate[:nrows].astype(np.float64))
    got = to_f64(y_perm[:nrows])
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            assert rel_err(got[lo:hi], ref[lo:hi]) <= TOL_BF16, "group of %d rows" % (hi - lo)
    # rows past the routed groups are never written
    assert not torch.any(y_perm[nrows:T * k]).item()
    if wl.d_ff_shared:
        sh_ref = oracle.expert_apply(dims, host["x"], weights_host(host), np.arange(T, dtype=np.int32),
                                     np.full(T, E, np.int32))
        assert rel_err(to_f64(y_perm[T * k:]), sh_ref) <= TOL_BF16


@pytest.mark.parametrize("wl", CASES, ids=lambda w: w.name)
def test_group_sizes_fp8(wl, cuda_device):
    """The same group sizes through the e4m3 grouped FFN (x quantized per row
    on the device, weights as e4m3 codes with per-channel scales), against
    the oracle's FP8 expert on the same codes."""
    dev = cuda_device
    inp = syn.generate(wl, dev, seed=21, weights=False)
    w8 = syn.generate_fp8_experts(wl, dev, seed=21)
    cfg = nat.config_from_workload(wl)
    T, k, E, d = wl.T, wl.top_k, wl.E, wl.d_model
    rng = np.random.default_rng(6)
    sizes = np.array(SIZES, np.int64)
    rng.shuffle(sizes)
    nrows = int(sizes.sum())
    offsets = np.zeros(E + 1, np.int32)
    offsets[1:] = np.cumsum(sizes)
    row_token = rng.integers(0, T, T * k).astype(np.int32)
    row_gate = rng.uniform(0.05, 1.0, T * k).astype(np.float32)
    x8 = torch.empty((T, d), dtype=torch.uint8, device=dev)
    xs = torch.empty(T, dtype=torch.float32, device=dev)
    nat.moe_quantize_rows_e4m3(inp["x"], x8, xs)
    rt = torch.from_numpy(row_token.astype(np.int64)).to(dev)
    x8_perm = x8[rt].contiguous()
    xps = xs[rt].contiguous()
    y_perm = torch.zeros((nat.perm_rows(cfg), d), dtype=torch.bfloat16, device=dev)
    ws = nat.alloc_workspace(cfg, dev)
    nat.moe_grouped_ffn_fp8(cfg, x8_perm, xps, torch.from_numpy(offsets).to(dev), torch.from_numpy(row_gate).to(dev),
                            w8, w8.get("b1"), w8.get("b2"), x8, xs, y_perm, ws)
    torch.cuda.synchronize(dev)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK

    dims = oracle_dims(wl)
    x8h, xsh = x8.cpu().numpy(), xs.cpu().numpy()
    rc, rs = oracle.quantize_rows(to_f64(inp["x"]).astype(np.float32))
    assert np.array_equal(x8h, rc) and np.array_equal(xsh, rs)
    w8h = {key: v.cpu().numpy() for key, v in w8.items() if v is not None}
    row_expert = np.repeat(np.arange(E), sizes).astype(np.int32)
    ref = oracle.expert_apply_fp8(dims, x8h, xsh, w8h, row_token[:nrows], row_expert,
                                  row_gate[:nrows].astype(np.float64))
    got = to_f64(y_perm[:nrows])
    for e in range(E):
        lo, hi = offsets[e], offsets[e + 1]
        if hi > lo:
            assert rel_err(got[lo:hi], ref[lo:hi]) <= TOL_BF16, "group of %d rows" % (hi - lo)
    assert not torch.any(y_perm[nrows:T * k]).item()
    if wl.d_ff_shared:
        sh_ref = oracle.expert_apply_fp8(dims, x8h, xsh, w8h, np.arange(T, dtype=np.int32), np.full(T, E, np.int32))
        assert rel_err(to_f64(y_perm[T * k:]), sh_ref) <= TOL_BF16
