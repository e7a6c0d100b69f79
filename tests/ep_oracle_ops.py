"""The expert-parallel layer's local steps computed by the CPU oracle (fp64),
for running the expert-parallel orchestration on CPU ranks.  Test
infrastructure: the same interface as expert_parallel.NativeOps, every step
through the oracle's functions on numpy arrays."""
import numpy as np
import torch

import oracle
from mixture_experts_layer_49_b200 import native as nat
from mixture_experts_layer_49_b200 import synthetic as syn


def dims_of(cfg, T=None, E=None, k=None, capacity=None):
    T = cfg.T if T is None else T
    E = cfg.E if E is None else E
    k = cfg.top_k if k is None else k
    if capacity is None:
        capacity = oracle.capacity(float(np.float32(cfg.capacity_factor)), cfg.top_k, cfg.T, cfg.E)
    return oracle.make_dims(T, cfg.d_model, E, cfg.d_ff, k,
                            x_dtype="bf16" if cfg.dtype == nat.MOE_BF16 else "f32",
                            act="swiglu" if cfg.act == nat.MOE_ACT_SWIGLU else "gelu",
                            score="sigmoid" if cfg.score == nat.MOE_SCORE_SIGMOID else "softmax",
                            renorm=cfg.renorm, capacity=capacity, d_ff_shared=cfg.d_ff_shared, nthreads=2)


def _np(t):
    return None if t is None else syn.to_numpy_raw(t)


def _weights(w):
    return {k: _np(w[k]) for k in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd") if w.get(k) is not None}


class OracleOps:
    def route(self, cfg, x, Wr, logit_bias, sel_bias):
        r = oracle.route(dims_of(cfg), _np(x), _np(Wr), _np(logit_bias), _np(sel_bias))
        # score sums in blocks of one token: the gathered blocks are the job's pnorm rows
        return torch.from_numpy(r["idx"]), torch.from_numpy(r["gate"]), torch.from_numpy(r["pnorm"])

    def permute(self, cfg, x, idx, gate):
        dp = oracle.dispatch(dims_of(cfg), idx.numpy())
        T, k = cfg.T, cfg.top_k
        n = int(dp["offsets"][-1])
        row_gate = torch.zeros(T * k, dtype=torch.float64)
        ro = torch.from_numpy(dp["row_of"])
        kept = ro >= 0
        row_gate[ro[kept].long()] = gate[kept]
        x_perm = torch.zeros((T * k, cfg.d_model), dtype=x.dtype)
        x_perm[:n] = x[torch.from_numpy(dp["row_token"]).long()]
        return dict(counts=torch.from_numpy(dp["counts"]), kept=torch.from_numpy(dp["kept"]),
                    offsets=torch.from_numpy(dp["offsets"]), row_of=ro, row_gate=row_gate, x_perm=x_perm,
                    n_dropped=torch.tensor([dp["n_dropped"]], dtype=torch.int32))

    def expert_ffn(self, cfg_local, n_src, group_offsets, x_rows, row_gate, w):
        offs = group_offsets.tolist()
        rows = x_rows.shape[0]
        el = cfg_local.E
        y = torch.zeros((rows, cfg_local.d_model), dtype=torch.float64)
        n = offs[-1]
        if n == 0:
            return y
        expert = np.zeros(n, np.int32)
        for g in range(n_src * el):
            expert[offs[g]:offs[g + 1]] = g % el
        dims = dims_of(cfg_local, T=rows, E=el, k=1, capacity=-1)
        y[:n] = torch.from_numpy(oracle.expert_apply(dims, _np(x_rows), _weights(w), np.arange(n, dtype=np.int32),
                                                     expert, row_gate[:n].numpy().astype(np.float64)))
        return y

    def shared_ffn(self, cfg_sh, x, w, x_perm, row_gate, y_perm):
        T, k = cfg_sh.T, cfg_sh.top_k
        dims = dims_of(cfg_sh, capacity=-1)
        out = oracle.expert_apply(dims, _np(x), _weights(w), np.arange(T, dtype=np.int32),
                                  np.full(T, cfg_sh.E, np.int32))
        y_perm[T * k:T * k + T] = torch.from_numpy(out)

    def combine(self, cfg, y_perm, row_of):
        T, k = cfg.T, cfg.top_k
        y = torch.zeros((T, cfg.d_model), dtype=torch.float64)
        for s in range(k):
            r = row_of[:, s]
            kept = r >= 0
            y[kept] += y_perm[r[kept].long()]
        if cfg.d_ff_shared > 0:
            y += y_perm[T * k:T * k + T]
        return y

    def balance(self, cfg_job, counts, psum):
        b = oracle.balance(dims_of(cfg_job), counts.numpy(), psum.numpy())
        return torch.from_numpy(b["f"]), torch.from_numpy(b["P"]), torch.tensor([b["loss"]], dtype=torch.float64)
