"""Expert parallelism on the GPU.

1. moe_ep_grouped_ffn through the C ABI on hand-made received layouts
   (several sources, empty groups, groups that straddle tile boundaries): every
   row against the oracle's expert (group g uses local expert g % E) with its
   gate, within the layer tolerances (bf16 2e-2, fp32 1e-4 of max|y_ref|).
2. The whole expert-parallel forward (expert_parallel.ep_forward with the
   libmoe steps) with R = 2 and 4 ranks emulated on one GPU: one host thread
   and one CUDA stream per rank, the all-to-alls done as device copies after
   the source rank's stream has synchronised (no kernel waits on another
   rank).  Each rank's routing, counts and dispatch equal the single-device
   forward pass on its tokens bit for bit, its y equals the oracle within the
   bf16 tolerance, and the job-wide loss equals the oracle's on the
   concatenated batch.
"""
import threading

import numpy as np
import pytest
import torch

import oracle
from mixture_experts_layer_49_b200 import expert_parallel as ep
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn

from helpers import TOL_BF16, TOL_F32, TOL_LOSS, check_routing, make_case, oracle_dims, rel_err, weights_host

pytestmark = pytest.mark.gpu


# ---------------------------------------------------------------- 1. the entry point
@pytest.mark.parametrize("dtype,act,sizes", [
    ("bf16", "swiglu", [[0, 130, 1, 257], [64, 0, 129, 3], [300, 17, 0, 128]]),
    ("bf16", "gelu", [[5, 256, 0, 2], [0, 0, 0, 513]]),
    ("f32", "gelu", [[3, 70, 0, 65], [1, 0, 129, 8], [40, 2, 2, 0]]),
], ids=["bf16_swiglu_3src", "bf16_gelu_2src", "f32_gelu_3src"])
def test_ep_grouped_ffn_rows_against_oracle(dtype, act, sizes, cuda_device):
    n_src, el = len(sizes), len(sizes[0])
    d, F = 256, 192
    wl = syn.Workload("ep_ffn", T=64, d_model=d, E=el, d_ff=F, top_k=1, dtype=dtype, act=act)
    inp = syn.generate(wl, cuda_device, seed=11)
    counts = [c for src in sizes for c in src]
    offs = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    n = int(offs[-1])
    max_rows = n + 37                                  # slack rows stay untouched
    dt = torch.bfloat16 if dtype == "bf16" else torch.float32
    g = torch.Generator(device=cuda_device).manual_seed(3)
    x_rows = torch.randn((max_rows, d), generator=g, device=cuda_device).to(dt)
    gate = torch.rand(max_rows, generator=g, device=cuda_device) + 0.1
    y = torch.full((max_rows, d), 7.0, dtype=dt, device=cuda_device)
    cfg = nat.make_config(0, d, el, F, 1, dtype=dtype, act=act)
    ws = torch.empty(nat.ep_workspace_size(cfg, n_src, max_rows), dtype=torch.uint8, device=cuda_device)
    nat.moe_workspace_init(ws)
    go = torch.from_numpy(offs).to(cuda_device)
    nat.moe_ep_grouped_ffn(cfg, n_src, go, x_rows, gate, inp["W1"], inp.get("b1"), inp.get("Wu"), inp["W2"],
                           inp.get("b2"), y, ws)
    assert nat.moe_get_device_status(ws) == nat.MOE_OK
    expert = np.zeros(n, np.int32)
    for grp in range(n_src * el):
        expert[offs[grp]:offs[grp + 1]] = grp % el
    dims = oracle.make_dims(max_rows, d, el, F, 1, x_dtype=dtype, act=act)
    w = {k: syn.to_numpy_raw(inp[k]) for k in ("W1", "Wu", "W2", "b1", "b2") if inp.get(k) is not None}
    ref = oracle.expert_apply(dims, syn.to_numpy_raw(x_rows), w, np.arange(n, dtype=np.int32), expert,
                              gate[:n].double().cpu().numpy())
    err = rel_err(y[:n].double().cpu().numpy(), ref)
    assert err <= (TOL_BF16 if dtype == "bf16" else TOL_F32), err
    assert torch.all(y[n:] == 7.0)


def test_ep_grouped_ffn_checks_arguments(cuda_device):
    cfg = nat.make_config(0, 64, 4, 64, 1)
    assert nat.lib().moe_ep_workspace_size(cfg, 65, 10) == 0          # 65 * 4 groups > 256
    x = torch.zeros((8, 64), dtype=torch.bfloat16, device=cuda_device)
    ws = torch.empty(256, dtype=torch.uint8, device=cuda_device)     # far too small for 8 rows
    offs = torch.zeros(9, dtype=torch.int32, device=cuda_device)
    w = torch.zeros((4, 64, 64), dtype=torch.bfloat16, device=cuda_device)
    with pytest.raises(nat.MoEError) as e:
        nat.moe_ep_grouped_ffn(cfg, 2, offs, x, torch.ones(8, device=cuda_device), w, None, w, w, None, x, ws)
    assert e.value.status == nat.MOE_ERR_WORKSPACE


# ---------------------------------------------------------------- 2. emulated ranks
class ThreadComm:
    """Collectives among R host threads of one process, one GPU: each rank
    synchronises its stream, publishes its tensor, and copies what it needs
    from the others' tensors after a barrier (no kernel ever waits on
    another rank's kernel)."""

    def __init__(self, shared, rank):
        self.s = shared
        self.rank = rank
        self.world = shared["world"]

    def _publish(self, item):
        torch.cuda.current_stream().synchronize()
        self.s["slots"][self.rank] = item
        self.s["barrier"].wait()

    def _done(self):
        torch.cuda.current_stream().synchronize()
        self.s["barrier"].wait()

    def all_to_all(self, out, inp, out_splits, in_splits):
        self._publish((inp, list(in_splits)))
        o = 0
        for src in range(self.world):
            sinp, ssplits = self.s["slots"][src]
            start, n = sum(ssplits[:self.rank]), ssplits[self.rank]
            assert n == out_splits[src]
            if n:
                out[o:o + n].copy_(sinp[start:start + n])
            o += n
        self._done()

    def all_gather_cat(self, t):
        self._publish(t)
        res = torch.cat([self.s["slots"][r] for r in range(self.world)], 0)
        self._done()
        return res

    def all_reduce_sum(self, t):
        self._publish(t.clone())
        acc = self.s["slots"][0].clone()
        for r in range(1, self.world):
            acc += self.s["slots"][r]
        self._done()
        t.copy_(acc)
        return t


def run_ranks(world, fn):
    shared = dict(world=world, barrier=threading.Barrier(world, timeout=120), slots=[None] * world)
    results, errors = [None] * world, []

    def body(rank):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                results[rank] = fn(rank, ThreadComm(shared, rank), stream)
                stream.synchronize()
        except BaseException as exc:             # noqa: BLE001 -- re-raised below
            errors.append(exc)
            shared["barrier"].abort()

    threads = [threading.Thread(target=body, args=(r,)) for r in range(world)]
    for th in threads:
        th.start()
    for th in threads:
        th.join()
    if errors:
        raise errors[0]
    return results


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("wl", [
    syn.Workload("ep_qwen_like", T=4 * 192, d_model=256, E=32, d_ff=128, top_k=4, logit_skew="zipf"),
    syn.Workload("ep_deepseek_like", T=4 * 128, d_model=256, E=16, d_ff=128, top_k=4, score="sigmoid",
                 sel_bias_std=0.1, d_ff_shared=96),
    syn.Workload("ep_switch_like", T=4 * 256, d_model=128, E=8, d_ff=256, top_k=1, act="gelu", renorm=0,
                 capacity_factor=1.0, logit_skew="normal"),
], ids=lambda w: w.name)
def test_expert_parallel_forward_emulated_ranks(wl, world, cuda_device):
    inp, host = make_case(wl, cuda_device, seed=4)       # the job's batch, selection margin enforced
    t_rank = wl.T // world

    def rank_fn(rank, comm, stream):
        lo, hi = ep.expert_range(wl.E, world, rank)
        w_local = {k: (inp[k][lo:hi].contiguous() if k in ("W1", "Wu", "W2", "b1", "b2") else inp[k])
                   for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd") if inp.get(k) is not None}
        x_mine = inp["x"][rank * t_rank:(rank + 1) * t_rank].contiguous()
        cfg = nat.config_from_workload(wl, T=t_rank)
        res = ep.ep_forward(cfg, x_mine, inp["Wr"], w_local, comm, ep.NativeOps(stream),
                            logit_bias=inp.get("logit_bias"), sel_bias=inp.get("sel_bias"))
        # the single-device layer on the same tokens, same stream
        out = nat.Outputs(cfg)
        ws = nat.alloc_workspace(cfg, stream=stream)
        inp_r = dict(inp)
        inp_r["x"] = x_mine
        nat.forward(cfg, inp_r, out, ws, stream)
        tab = nat.workspace_tables(cfg, ws)
        stream.synchronize()
        return dict(res=res, out=out, row_of=tab["row_of"].clone(), status=nat.moe_get_device_status(ws, stream))

    results = run_ranks(world, rank_fn)
    job_dims = oracle_dims(wl)
    r_all = oracle.route(job_dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"])
    for rank, rr in enumerate(results):
        res, out = rr["res"], rr["out"]
        assert rr["status"] == nat.MOE_OK
        assert torch.equal(res.idx, out.idx) and torch.equal(res.gate, out.gate)
        assert torch.equal(res.counts, out.counts) and torch.equal(res.row_of, rr["row_of"])
        sl = slice(rank * t_rank, (rank + 1) * t_rank)
        ref_r = dict(idx=r_all["idx"][sl], gate=r_all["gate"][sl], sel_key=r_all["sel_key"][sl])
        check_routing(res.idx.cpu().numpy(), res.gate.cpu().numpy(), ref_r)
        dims_r = oracle_dims(wl.replace(T=t_rank))
        ridx = np.ascontiguousarray(r_all["idx"][sl])
        dp = oracle.dispatch(dims_r, ridx)
        y_ref = oracle.layer_tokens(dims_r, np.ascontiguousarray(host["x"][sl]), weights_host(host), ridx,
                                    np.ascontiguousarray(r_all["gate"][sl]), dp["row_of"],
                                    np.arange(t_rank, dtype=np.int32))
        err = rel_err(res.y.double().cpu().numpy(), y_ref)
        assert err <= TOL_BF16, (rank, err)
        # the same rows through the same kernels: the expert-parallel y equals
        # the single-device y to within one bf16 rounding of the gated rows
        assert rel_err(res.y.double().cpu().numpy(), out.y.double().cpu().numpy()) <= 1e-2
    counts_job = np.bincount(r_all["idx"].ravel(), minlength=wl.E).astype(np.int32)
    bal = oracle.balance(job_dims, counts_job, r_all["pnorm"])
    for rr in results:
        assert abs(float(rr["res"].loss.item()) - bal["loss"]) <= TOL_LOSS * bal["loss"]
        np.testing.assert_array_equal(rr["res"].f.cpu().numpy(), results[0]["res"].f.cpu().numpy())
