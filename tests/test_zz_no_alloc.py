"""moe_permute_noalloc: the permutation for callers that cannot allocate
device memory (a plug-in inside a framework that owns the device-memory
budget, or a caller that cannot take cudaMalloc's implicit synchronisation).

It keeps its scratch in a fixed array inside libmoe instead of a caller
workspace.  Called through the C ABI, its outputs must equal those of
moe_permute (the entry point with a workspace) exactly -- this is integer and
copy work, so the tests' tolerance is bit-exactness -- and the oracle's
dispatch of the same expert ids.  The calls run back to back without
reloading the library: two calls of one shape with different inputs, then a
smaller and a larger problem, so nothing a call leaves in the shared array
reaches the next one.  The row-tables-only form (x_perm NULL) is checked too.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import oracle_dims

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


def call_noalloc_raw(cfg, x, idx, gate, o, with_rows=True):
    """Straight through the C ABI (ctypes), no workspace argument."""
    L = nat.lib()
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return L.moe_permute_noalloc(ctypes.byref(cfg), p(x), p(idx), p(gate), p(o["counts"]), p(o["kept"]),
                                 p(o["offsets"]), p(o["row_of"]), p(o["row_token"]), p(o["row_gate"]),
                                 p(o["x_perm"]) if with_rows else None, p(o["n_dropped"]), stream)


def check_one_call(wl, dev, seed, with_rows=True):
    cfg, x, idx, gate, ws = routing(wl, dev, seed)
    ref = permute_outputs(wl, dev)
    nat.moe_permute(cfg, x, idx, gate, ref["counts"], ref["kept"], ref["offsets"], ref["row_of"],
                    ref["row_token"], ref["row_gate"], ref["x_perm"] if with_rows else None, ref["n_dropped"], ws)
    got = permute_outputs(wl, dev)
    rc = call_noalloc_raw(cfg, x, idx, gate, got, with_rows)
    assert rc == nat.MOE_OK, nat.last_error_detail()
    torch.cuda.synchronize()
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    nrows = int(ref["offsets"][-1].item())
    # against the entry point with a workspace
    for key in ("counts", "kept", "offsets", "row_of", "n_dropped"):
        assert torch.equal(got[key], ref[key]), (seed, key)
    for key in ("row_token", "row_gate"):
        assert torch.equal(got[key][:nrows], ref[key][:nrows]), (seed, key)
    if with_rows:
        assert torch.equal(got["x_perm"][:nrows], ref["x_perm"][:nrows]), seed
    else:
        assert int(torch.count_nonzero(got["x_perm"]).item()) == 0    # untouched
    # against the oracle's dispatch of the same expert ids
    dp = oracle.dispatch(oracle_dims(wl), idx.cpu().numpy())
    np.testing.assert_array_equal(got["counts"].cpu().numpy(), dp["counts"])
    np.testing.assert_array_equal(got["kept"].cpu().numpy(), dp["kept"])
    np.testing.assert_array_equal(got["offsets"].cpu().numpy(), dp["offsets"])
    np.testing.assert_array_equal(got["row_of"].cpu().numpy(), dp["row_of"])
    np.testing.assert_array_equal(got["row_token"][:nrows].cpu().numpy(), dp["row_token"])
    assert int(got["n_dropped"].item()) == dp["n_dropped"]
    if with_rows:
        tok = got["row_token"][:nrows].long()
        assert torch.equal(got["x_perm"][:nrows], x[tok])
    return int(got["n_dropped"].item())


CAPPED = syn.Workload("noalloc_cap", T=2000, d_model=256, E=32, d_ff=64, top_k=4, capacity_factor=0.8,
                      logit_skew="zipf")
F32 = syn.Workload("noalloc_f32", T=777, d_model=96, E=8, d_ff=64, top_k=2, dtype="f32", logit_skew="normal")
WIDE = syn.Workload("noalloc_wide", T=5000, d_model=128, E=64, d_ff=64, top_k=6, logit_skew="zipf")


@pytest.mark.parametrize("wl", [CAPPED, F32], ids=lambda w: w.name)
def test_noalloc_matches_workspace_permute_twice(wl, cuda_device):
    for seed in (21, 22):                            # two calls in a row, different inputs
        dropped = check_one_call(wl, cuda_device, seed)
        if wl.capacity_factor > 0:
            assert dropped > 0


def test_noalloc_sizes_change_between_calls(cuda_device):
    # the count planes move when E * ceil(T/64) changes: a large problem, a
    # small one, then the large one again, with no reload in between
    for wl, seed in ((WIDE, 31), (F32, 32), (CAPPED, 33), (WIDE, 34)):
        check_one_call(wl, cuda_device, seed)


def test_noalloc_row_tables_only(cuda_device):
    check_one_call(CAPPED, cuda_device, 41, with_rows=False)


def test_noalloc_rejects_problems_beyond_its_scratch(cuda_device):
    # E * ceil(T / 64) = 256 * 1025 cells > 262144: refused before any launch
    wl = syn.Workload("too_big", T=65600, d_model=64, E=256, d_ff=64, top_k=1)
    cfg = nat.config_from_workload(wl)
    dummy = torch.zeros(64, dtype=torch.int32, device=cuda_device)
    p = ctypes.c_void_p(dummy.data_ptr())
    rc = nat.lib().moe_permute_noalloc(ctypes.byref(cfg), *([p] * 11), None)
    assert rc == nat.MOE_ERR_UNSUPPORTED
    assert "static scratch" in nat.last_error_detail()
