"""Expert parallelism: the MoE layer forward with its experts sharded over the
ranks of a process group.

The pages' distributed recipe ("Fine-Tuning Mixture of Experts (MoE) Models:
Router Optimization Techniques", Why It Matters 2, token dispatch and gather,
and Architecture & Distributed Execution; "Mixture-of-Experts", Vector
Institute post, expert-parallelism paragraph): each of R ranks holds E / R of
the experts; tokens are routed where they live, travel to the rank of each
expert they chose, pass through it there and travel back to be combined.

One rank's forward pass (rank r of R, its own T_r tokens, E_l = E / R local
experts, experts [r E_l, (r+1) E_l)):
  1. moe_router_topk and moe_permute on the local tokens over all E experts:
     rows come out in (expert, token) order, so the rows bound for rank j are
     the contiguous block of j's experts.
  2. The kept counts are exchanged (an all-to-all of E_l counts per rank
     pair), giving every rank the size of each (source, local expert) group.
  3. The rows and their gates travel to their experts' ranks (an all-to-all
     of variable-size blocks).  A rank receives n_src = R blocks, block src
     holding src's rows for local expert 0, 1, .., E_l - 1.
  4. moe_ep_grouped_ffn runs the local experts over the R * E_l groups
     (group src * E_l + e uses local expert e) with the gate applied.
  5. The gated rows travel back (the reverse all-to-all) into the source
     rank's own row order; the shared expert, if any, runs locally
     (moe_grouped_ffn with no routed rows); moe_combine sums them per token.
  6. Balance statistics over the whole job's batch: the per-expert counts
     are summed over ranks (all-reduce) and the router's per-block score sums
     gathered (all-gather), then moe_balance_stats on the job's batch.

Capacity: each rank's tokens form one capacity group (the per-expert
capacity floor(c k T_r / E) is applied to the rank's own batch), so rank r's
outputs equal the single-device layer applied to rank r's tokens.  The job's
balance statistics need every rank to hold the same number of tokens, a
multiple of the router's score-sum block (64 tokens for bf16 layers, 32 for
fp32 layers), so that the gathered blocks are those of the job's batch.

The collectives are torch.distributed calls (NCCL between GPUs, gloo for
CPU ranks) behind a small communicator interface; the compute steps are
libmoe entry points behind an `ops` interface (NativeOps here), so the same
orchestration runs with another communicator or another implementation of
the steps.  No multicast and no peer loads are used: remote rows land in
local memory before any kernel reads them.
"""
from __future__ import annotations

import dataclasses

import torch

from . import native as nat


# ---------------------------------------------------------------- communicators
class TorchComm:
    """Collectives of a torch.distributed process group (NCCL or gloo)."""

    def __init__(self, group=None):
        import torch.distributed as dist
        self.dist = dist
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)

    def all_to_all(self, out, inp, out_splits, in_splits):
        """Block i of `inp` (in_splits[i] rows) goes to rank i; block j of
        `out` (out_splits[j] rows) comes from rank j."""
        self.dist.all_to_all_single(out, inp, list(out_splits), list(in_splits), group=self.group)

    def all_gather_cat(self, t):
        """Concatenation over ranks (rank order) of equal-shape tensors."""
        parts = [torch.empty_like(t) for _ in range(self.world)]
        self.dist.all_gather(parts, t.contiguous(), group=self.group)
        return torch.cat(parts, 0)

    def all_reduce_sum(self, t):
        self.dist.all_reduce(t, group=self.group)
        return t


# ---------------------------------------------------------------- local steps
class NativeOps:
    """The layer's local steps through libmoe (device tensors, one stream)."""

    def __init__(self, stream=None):
        self.stream = stream
        self._ws = {}

    def _workspace(self, key, nbytes, device):
        ws = self._ws.get(key)
        if ws is None or ws.numel() < nbytes:
            ws = torch.empty(max(nbytes, 256), dtype=torch.uint8, device=device)
            nat.moe_workspace_init(ws, stream=self.stream)
            self._ws[key] = ws
        return ws

    def route(self, cfg, x, Wr, logit_bias, sel_bias):
        dev = x.device
        ws = self._workspace("layer", nat.workspace_size(cfg), dev)
        idx = torch.empty((cfg.T, cfg.top_k), dtype=torch.int32, device=dev)
        gate = torch.empty((cfg.T, cfg.top_k), dtype=torch.float32, device=dev)
        psum = torch.empty((nat.router_blocks(cfg), cfg.E), dtype=torch.float32, device=dev)
        nat.moe_router_topk(cfg, x, Wr, logit_bias, sel_bias, idx, gate, None, psum, ws, self.stream)
        return idx, gate, psum

    def permute(self, cfg, x, idx, gate):
        dev = x.device
        ws = self._workspace("layer", nat.workspace_size(cfg), dev)
        T, E, k = cfg.T, cfg.E, cfg.top_k
        o = dict(counts=torch.empty(E, dtype=torch.int32, device=dev),
                 kept=torch.empty(E, dtype=torch.int32, device=dev),
                 offsets=torch.empty(E + 1, dtype=torch.int32, device=dev),
                 row_of=torch.empty((T, k), dtype=torch.int32, device=dev),
                 row_token=torch.empty(T * k, dtype=torch.int32, device=dev),
                 row_gate=torch.empty(T * k, dtype=torch.float32, device=dev),
                 x_perm=torch.empty((T * k, cfg.d_model), dtype=x.dtype, device=dev),
                 n_dropped=torch.zeros(1, dtype=torch.int32, device=dev))
        nat.moe_permute(cfg, x, idx, gate, o["counts"], o["kept"], o["offsets"], o["row_of"], o["row_token"],
                        o["row_gate"], o["x_perm"], o["n_dropped"], ws, self.stream)
        return o

    def expert_ffn(self, cfg_local, n_src, group_offsets, x_rows, row_gate, w):
        rows = x_rows.shape[0]
        ws = self._workspace("ep", nat.ep_workspace_size(cfg_local, n_src, rows), x_rows.device)
        y_rows = torch.empty_like(x_rows)
        nat.moe_ep_grouped_ffn(cfg_local, n_src, group_offsets, x_rows, row_gate, w["W1"], w.get("b1"),
                               w.get("Wu"), w["W2"], w.get("b2"), y_rows, ws, self.stream)
        return y_rows

    def shared_ffn(self, cfg_sh, x, w, x_perm, row_gate, y_perm):
        """The shared expert over every local token, written to the shared
        rows T*k + t of y_perm (the call has no routed rows)."""
        ws = self._workspace("shared", nat.workspace_size(cfg_sh), x.device)
        zero = torch.zeros(cfg_sh.E + 1, dtype=torch.int32, device=x.device)
        nat.moe_grouped_ffn(cfg_sh, x_perm, zero, row_gate, w["W1"], w.get("b1"), w.get("Wu"), w["W2"],
                            w.get("b2"), x, w["Wsg"], w.get("Wsu"), w["Wsd"], y_perm, ws, self.stream)

    def combine(self, cfg, y_perm, row_of):
        y = torch.empty((cfg.T, cfg.d_model), dtype=y_perm.dtype, device=y_perm.device)
        ws = self._workspace("layer", nat.workspace_size(cfg), y_perm.device)
        nat.moe_combine(cfg, y_perm, row_of, y, ws, self.stream)
        return y

    def balance(self, cfg_job, counts, psum):
        """Statistics of the job's batch from the ranks' gathered score-sum
        blocks (rank order), which are the job batch's own blocks when every
        rank holds the same multiple of the block size."""
        if psum.shape[0] != nat.router_blocks(cfg_job):
            raise ValueError("job-wide statistics need every rank to hold the same number of tokens, a "
                             "multiple of the router's score-sum block (%d blocks gathered for %d tokens)"
                             % (psum.shape[0], cfg_job.T))
        dev = counts.device
        f = torch.empty(cfg_job.E, dtype=torch.float32, device=dev)
        P = torch.empty(cfg_job.E, dtype=torch.float32, device=dev)
        loss = torch.empty(1, dtype=torch.float64, device=dev)
        nat.moe_balance_stats(cfg_job, counts, psum, f, P, loss, self.stream)
        return f, P, loss

    def synchronize(self, device):
        torch.cuda.synchronize(device)


# ---------------------------------------------------------------- the layer
@dataclasses.dataclass
class EPResult:
    y: torch.Tensor                 # [T_r, d_model] this rank's outputs
    idx: torch.Tensor               # [T_r, k] chosen experts (global ids)
    gate: torch.Tensor              # [T_r, k]
    counts: torch.Tensor            # [E] this rank's assignments per expert (before capacity)
    kept: torch.Tensor              # [E]
    row_of: torch.Tensor            # [T_r, k] local row of each assignment, -1 when dropped
    send_rows: list                 # rows sent to each rank
    recv_rows: list                 # rows received from each rank
    recv_kept: torch.Tensor         # [R, E_l] rows received per (source, local expert)
    f: torch.Tensor = None          # [E] job-wide statistics (when computed)
    P: torch.Tensor = None
    loss: torch.Tensor = None


def expert_range(E, world, rank):
    """Experts held by `rank`: [rank * E/R, (rank+1) * E/R)."""
    if E % world:
        raise ValueError("E = %d experts do not divide over %d ranks" % (E, world))
    el = E // world
    return rank * el, (rank + 1) * el


def local_config(cfg, world):
    """moe_config of this rank's expert shard (for moe_ep_grouped_ffn)."""
    el = cfg.E // world
    return nat.make_config(cfg.T, cfg.d_model, el, cfg.d_ff, 1,
                           dtype="bf16" if cfg.dtype == nat.MOE_BF16 else "f32",
                           act="swiglu" if cfg.act == nat.MOE_ACT_SWIGLU else "gelu")


def shared_config(cfg, world):
    """Config of the shared-expert-only call: E = E_l local experts (no routed
    rows), the rank's T tokens and top_k, so the shared rows land at T*k + t."""
    el = cfg.E // world
    if cfg.top_k > el:
        raise ValueError("a shared expert needs top_k <= E / R (%d > %d)" % (cfg.top_k, el))
    c = nat.MoeConfig()
    for name, _ in nat.MoeConfig._fields_:
        setattr(c, name, getattr(cfg, name))
    c.E = el
    c.capacity_factor = 0.0
    return c


def ep_forward(cfg, x, Wr, local_w, comm, ops, logit_bias=None, sel_bias=None, job_stats=True):
    """One rank's part of the expert-parallel forward pass.

    cfg: moe_config of the rank's own batch (T = this rank's tokens, E = all
    experts).  local_w: this rank's expert slices W1, Wu, W2 [E_l, ...], b1,
    b2, and the (replicated) shared expert Wsg, Wsu, Wsd.  Returns EPResult."""
    R, r = comm.world, comm.rank
    E, k, d = cfg.E, cfg.top_k, cfg.d_model
    e_lo, e_hi = expert_range(E, R, r)
    el = e_hi - e_lo
    T = cfg.T

    # 1. local routing and permutation over all experts
    idx, gate, psum = ops.route(cfg, x, Wr, logit_bias, sel_bias)
    p = ops.permute(cfg, x, idx, gate)

    # 2. kept counts: rank j gets this rank's counts for j's experts
    kept_dev = p["kept"]
    recv_kept = torch.empty_like(kept_dev)
    comm.all_to_all(recv_kept, kept_dev, [el] * R, [el] * R)
    kept_h = kept_dev.cpu().tolist()
    recv_h = recv_kept.cpu().tolist()
    send_rows = [sum(kept_h[j * el:(j + 1) * el]) for j in range(R)]
    recv_rows = [sum(recv_h[s * el:(s + 1) * el]) for s in range(R)]
    n_send, n_recv = sum(send_rows), sum(recv_rows)

    # 3. rows and gates to their experts' ranks
    x_recv = torch.empty((max(n_recv, 1), d), dtype=x.dtype, device=x.device)
    g_recv = torch.empty(max(n_recv, 1), dtype=p["row_gate"].dtype, device=x.device)
    comm.all_to_all(x_recv[:n_recv], p["x_perm"][:n_send], recv_rows, send_rows)
    comm.all_to_all(g_recv[:n_recv], p["row_gate"][:n_send], recv_rows, send_rows)

    # 4. the local experts over the received groups (source-major, expert-minor)
    offs = [0]
    for v in recv_h:
        offs.append(offs[-1] + v)
    group_offsets = torch.tensor(offs, dtype=torch.int32).to(x.device)
    y_recv = ops.expert_ffn(local_config(cfg, R), R, group_offsets, x_recv[:max(n_recv, 1)],
                            g_recv[:max(n_recv, 1)], local_w)

    # 5. back to the source ranks, in their own row order; shared expert; combine
    rows_total = T * k + (T if cfg.d_ff_shared > 0 else 0)
    y_perm = torch.empty((max(rows_total, 1), d), dtype=y_recv.dtype, device=x.device)
    comm.all_to_all(y_perm[:n_send], y_recv[:n_recv], send_rows, recv_rows)
    if cfg.d_ff_shared > 0 and T > 0:
        ops.shared_ffn(shared_config(cfg, R), x, local_w, p["x_perm"], p["row_gate"], y_perm)
    y = ops.combine(cfg, y_perm[:rows_total], p["row_of"])

    res = EPResult(y=y, idx=idx, gate=gate, counts=p["counts"], kept=kept_dev, row_of=p["row_of"],
                   send_rows=send_rows, recv_rows=recv_rows, recv_kept=recv_kept.view(R, el))

    # 6. job-wide balance statistics
    if job_stats:
        counts_job = comm.all_reduce_sum(p["counts"].clone())
        psum_job = comm.all_gather_cat(psum)
        cfg_job = nat.MoeConfig()
        for name, _ in nat.MoeConfig._fields_:
            setattr(cfg_job, name, getattr(cfg, name))
        cfg_job.T = T * R
        res.f, res.P, res.loss = ops.balance(cfg_job, counts_job, psum_job)
    return res
