"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (a plug-in inside a framework that owns the device-memory
budget, or a caller that cannot take cudaMalloc's implicit synchronisation).

It keeps its scratch in a fixed array inside libmoe instead of a caller
workspace.  Called through the C ABI, its outputs must equal those of
moe_permute (the entry point with a workspace) exactly -- this is integer and
copy work, so the tests' tolerance is bit-exactness -- on two calls in a row
with different inputs, so nothing from the first call leaks into the second.
"""
import ctypes

import pytest
import torch

from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

pytestmark = pytest.mark.gpu


def permute_outputs(wl, dev):
    T, d, E, k = wl.T, wl.d_model, wl.E, wl.top_k
    dt = torch.bfloat16 if wl.dtype == "bf16" else torch.float32
    return dict(counts=torch.full((E,), -7, dtype=torch.int32, device=dev),
                kept=torch.full((E,), -7, dtype=torch.int32, device=dev),
                offsets=torch.full((E + 1,), -7, dtype=torch.int32, device=dev),
                row_of=torch.full((T, k), -7, dtype=torch.int32, device=dev),
                row_token=torch.full((T * k,), -7, dtype=torch.int32, device=dev),
                row_gate=torch.full((T * k,), -7.0, dtype=torch.float32, device=dev),
                x_perm=torch.zeros((T * k, d), dtype=dt, device=dev),
                n_dropped=torch.full((1,), -7, dtype=torch.int32, device=dev))


def routing(wl, dev, seed):
    """Expert ids and gates from the library's own router."""
    inp = syn.generate(wl, dev, seed=seed, weights=False)
    cfg = nat.config_from_workload(wl)
    ws = nat.alloc_workspace(cfg, dev)
    idx = torch.empty((wl.T, wl.top_k), dtype=torch.int32, device=dev)
    gate = torch.empty((wl.T, wl.top_k), dtype=torch.float32, device=dev)
    psum = torch.empty((nat.router_blocks(cfg), wl.E), dtype=torch.float32, device=dev)
    nat.moe_router_topk(cfg, inp["x"], inp["Wr"], inp["logit_bias"], inp["sel_bias"], idx, gate, None, psum, ws)
    return cfg, inp["x"], idx, gate, ws


def call_noalloc_raw(cfg, x, idx, gate, o):
    """Straight through the C ABI (ctypes), no workspace argument."""
    L = nat.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.moe_permute_noalloc(ctypes.byref(cfg), p(x), p(idx), p(gate), p(o["counts"]), p(o["kept"]),
                                 p(o["offsets"]), p(o["row_of"]), p(o["row_token"]), p(o["row_gate"]),
                                 p(o["x_perm"]), p(o["n_dropped"]), stream)


@pytest.mark.parametrize("wl", [
    syn.Workload("noalloc_cap", T=2000, d_model=256, E=32, d_ff=64, top_k=4, capacity_factor=0.8,
                 logit_skew="zipf"),
    syn.Workload("noalloc_f32", T=777, d_model=96, E=8, d_ff=64, top_k=2, dtype="f32", logit_skew="normal"),
], ids=lambda w: w.name)
def test_noalloc_matches_workspace_permute_twice(wl, cuda_device):
    for call, seed in enumerate((21, 22)):           # two calls in a row, different inputs
        cfg, x, idx, gate, ws = routing(wl, cuda_device, seed)
        ref = permute_outputs(wl, cuda_device)
        nat.moe_permute(cfg, x, idx, gate, ref["counts"], ref["kept"], ref["offsets"], ref["row_of"],
                        ref["row_token"], ref["row_gate"], ref["x_perm"], ref["n_dropped"], ws)
        got = permute_outputs(wl, cuda_device)
        rc = call_noalloc_raw(cfg, x, idx, gate, got)
        assert rc == nat.MOE_OK, nat.last_error_detail()
        torch.cuda.synchronize()
        assert nat.moe_get_device_status(ws) == nat.MOE_OK
        nrows = int(ref["offsets"][-1].item())
        for key in ("counts", "kept", "offsets", "row_of", "n_dropped"):
            assert torch.equal(got[key], ref[key]), (call, key)
        for key in ("row_token", "row_gate", "x_perm"):
            assert torch.equal(got[key][:nrows], ref[key][:nrows]), (call, key)
        if wl.capacity_factor > 0:
            assert int(ref["n_dropped"].item()) > 0


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # E * ceil(T / 64) = 256 * 1025 cells > 262144: refused before any launch
    wl = syn.Workload("too_big", T=65600, d_model=64, E=256, d_ff=64, top_k=1)
    cfg = nat.config_from_workload(wl)
    dummy = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = nat.lib().moe_permute_noalloc(ctypes.byref(cfg), *([p] * 11), None)
    assert rc == nat.MOE_ERR_UNSUPPORTED
    assert "static scratch" in nat.last_error_detail()
