"""Expert-parallel orchestration on CPU ranks (gloo, world sizes 2 and 4).

Every rank holds E / R experts; the layer's local steps are the oracle's
(tests/ep_oracle_ops.py), the collectives are real torch.distributed calls.
What is checked is everything the orchestration decides: the kept-count
exchange, the send and receive splits, the group offsets of the received
rows and the expert each group uses, the return path into each source's row
order, the shared expert, the combine and the job-wide statistics.

Each rank's outputs must equal the single-process oracle on that rank's
tokens (each rank's batch is one capacity group): expert ids, gates and
counts bit for bit, y to 1e-12 of max|y|.  The job-wide f, P and loss must
equal the oracle's statistics of the concatenated batch to 1e-12.
"""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


WORKLOADS = {
    # name: (workload kwargs, tokens per rank)
    "swiglu_zipf": (dict(d_model=64, E=8, d_ff=48, top_k=2, logit_skew="zipf"), 40),
    "gelu_capacity": (dict(d_model=48, E=8, d_ff=32, top_k=2, act="gelu", renorm=0, capacity_factor=0.6,
                           logit_skew="normal"), 36),
    "sigmoid_shared": (dict(d_model=64, E=16, d_ff=32, top_k=4, score="sigmoid", sel_bias_std=0.1,
                            d_ff_shared=40), 30),
}


def _rank_main(rank, world, port, name, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, ROOT)
    sys.path.insert(0, HERE)
    import oracle
    from ep_oracle_ops import OracleOps, dims_of
    from mixture_experts_layer_49_b200 import expert_parallel as ep
    from mixture_experts_layer_49_b200 import native as nat
    from mixture_experts_layer_49_b200 import synthetic as syn

    kw, t_rank = WORKLOADS[name]
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        job = syn.Workload(name, T=t_rank * world, dtype="f32", **kw)
        inp = syn.generate(job, "cpu", seed=5)            # the same draws on every rank
        x_mine = inp["x"][rank * t_rank:(rank + 1) * t_rank].contiguous()
        lo, hi = ep.expert_range(job.E, world, rank)
        w_local = {k: (inp[k][lo:hi].contiguous() if k in ("W1", "Wu", "W2", "b1", "b2") else inp[k])
                   for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd") if inp.get(k) is not None}
        cfg = nat.config_from_workload(job, T=t_rank)
        comm = ep.TorchComm()
        res = ep.ep_forward(cfg, x_mine, inp["Wr"], w_local, comm, OracleOps(),
                            logit_bias=inp.get("logit_bias"), sel_bias=inp.get("sel_bias"))

        # single-process oracle on this rank's tokens
        host = {k: syn.to_numpy_raw(v) for k, v in inp.items() if isinstance(v, torch.Tensor)}
        weights = {k: host[k] for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd") if k in host}
        ref = oracle.forward(dims_of(cfg), syn.to_numpy_raw(x_mine), host["Wr"], weights,
                             logit_bias=host.get("logit_bias"), sel_bias=host.get("sel_bias"))
        np.testing.assert_array_equal(res.idx.numpy(), ref["idx"])
        np.testing.assert_array_equal(res.gate.numpy(), ref["gate"])
        np.testing.assert_array_equal(res.counts.numpy(), ref["counts"])
        np.testing.assert_array_equal(res.kept.numpy(), ref["kept"])
        np.testing.assert_array_equal(res.row_of.numpy(), ref["row_of"])
        y = res.y.numpy()
        err = np.max(np.abs(y - ref["y"])) / np.max(np.abs(ref["y"]))
        assert err <= 1e-12, err

        # job-wide statistics against the oracle over the concatenated batch
        job_dims = dims_of(nat.config_from_workload(job))
        r_all = oracle.route(job_dims, host["x"], host["Wr"], host.get("logit_bias"), host.get("sel_bias"))
        counts_all = np.bincount(r_all["idx"].ravel(), minlength=job.E).astype(np.int32)
        bal = oracle.balance(job_dims, counts_all, r_all["pnorm"])
        np.testing.assert_allclose(res.f.numpy(), bal["f"], rtol=1e-12)
        np.testing.assert_allclose(res.P.numpy(), bal["P"], rtol=1e-12)
        assert abs(float(res.loss[0]) - bal["loss"]) <= 1e-12 * bal["loss"]

        # the exchange itself: what this rank sent j is what j says it received
        sent = torch.tensor(res.send_rows, dtype=torch.int64)
        all_sent = [torch.empty_like(sent) for _ in range(world)]
        dist.all_gather(all_sent, sent)
        for src in range(world):
            assert int(all_sent[src][rank]) == res.recv_rows[src]
        assert sum(res.send_rows) == int(ref["offsets"][-1])
        out[rank] = dict(err=float(err), recv=list(res.recv_rows), send=list(res.send_rows))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("name", sorted(WORKLOADS))
def test_expert_parallel_matches_single_process(name, world):
    if WORKLOADS[name][0]["E"] % world:
        pytest.skip("experts do not divide over the ranks")
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_rank_main, args=(world, port, name, out), nprocs=world, join=True)
    assert sorted(out.keys()) == list(range(world))
    # every rank both sent and received rows (the experts really are remote)
    assert all(sum(out[r]["send"]) > 0 and sum(out[r]["recv"]) > 0 for r in range(world))
