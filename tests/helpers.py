"""Shared test plumbing: seeded cases with the selection margin enforced,
oracle dimensions for a workload, and the comparison measures.

The margin rule: for every token the key of its k-th choice must beat the
(k+1)-th by at least 1e-3 (keys computed by the fp64 oracle), so the fp32
GPU router and the fp64 oracle make the same selection.  Offending tokens get
fresh x rows from a seeded sub-stream until none is left.
"""
import numpy as np
import torch

import oracle
from mixture_experts_layer_49_b200 import synthetic as syn

MARGIN = 1e-3
TOL_BF16 = 2e-2      # max|y - y_ref| / max|y_ref| for bf16 layers
TOL_F32 = 1e-4       # the same measure for fp32 layers
TOL_LOSS = 1e-5      # relative error of the balance loss
TOL_GATE = 1e-5      # absolute error of an fp32 gate against the fp64 oracle
TIE_KEY = 1e-4       # selected experts whose keys differ by less than this may
                     # appear in either slot order (10x below the 1e-3 selection margin)
# Router logits, max|h - h_ref| / max|h_ref|.  bf16 layers compute them on the
# tensor cores: exact bf16 products (W_r split into three bf16 terms) but an
# fp32 accumulator that rounds toward zero at each K=16 step.  With S steps per
# accumulator the bias is bounded by about S * 2^-23 of the partial sum; the
# widest layer (d_model = 7168, E = 256: 2 accumulators, S = 672) bounds it at
# 8e-5 and measures 1.2e-5.  fp32 layers (FFMA router) stay far below 1e-6.
TOL_LOGIT = 5e-5

WEIGHT_KEYS = ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd")


def oracle_dims(wl, nthreads=None):
    # the layer takes the capacity factor as an fp32 value
    cap = oracle.capacity(float(np.float32(wl.capacity_factor)), wl.top_k, wl.T, wl.E)
    return oracle.make_dims(wl.T, wl.d_model, wl.E, wl.d_ff, wl.top_k, x_dtype=wl.dtype,
                            act=wl.act, score=wl.score, renorm=wl.renorm, capacity=cap,
                            d_ff_shared=wl.d_ff_shared, nthreads=nthreads)


def to_host(inp):
    h = {}
    for key in ("x", "Wr", "logit_bias", "sel_bias") + WEIGHT_KEYS:
        t = inp.get(key)
        h[key] = None if t is None else syn.to_numpy_raw(t)
    return h


def enforce_margin(wl, inp, host, seed, margin=MARGIN, max_rounds=100):
    dims = oracle_dims(wl)
    tokens = None
    for attempt in range(max_rounds):
        r = oracle.route(dims, host["x"], host["Wr"], host["logit_bias"], host["sel_bias"],
                         tokens=tokens, want_pnorm=False)
        rows = np.arange(wl.T) if tokens is None else tokens
        bad = rows[r["margin"] < margin]
        if len(bad) == 0:
            return attempt
        syn.redraw_rows(inp["x"], torch.from_numpy(bad.astype(np.int64)), wl, seed, attempt)
        host["x"][bad] = syn.to_numpy_raw(inp["x"][torch.from_numpy(bad.astype(np.int64)).to(inp["x"].device)])
        tokens = bad.astype(np.int32)
    raise RuntimeError("selection margin not reached after %d rounds" % max_rounds)


def make_case(wl, device, seed=0, margin=MARGIN):
    inp = syn.generate(wl, device, seed)
    host = to_host(inp)
    if wl.T > 0 and wl.top_k < wl.E:
        enforce_margin(wl, inp, host, seed, margin)
    return inp, host


def weights_host(host):
    return {k: host[k] for k in WEIGHT_KEYS if host.get(k) is not None}


def rel_err(y, ref):
    y = np.asarray(y, np.float64)
    ref = np.asarray(ref, np.float64)
    scale = np.max(np.abs(ref)) if ref.size else 0.0
    if ref.size == 0:
        return 0.0
    return float(np.max(np.abs(y - ref)) / max(scale, 1e-30))


def to_f64(t: torch.Tensor):
    return t.detach().to("cpu", torch.float64).numpy()


def sample_tokens(idx, row_of, E, n_random, seed, T):
    """Tokens for sampled output checks: the first and last token, n_random
    seeded draws, and for every expert with a kept row one token routed to it."""
    rng = np.random.default_rng(seed)
    chosen = {0, T - 1}
    chosen.update(rng.choice(T, size=min(n_random, T), replace=False).tolist())
    covered = set()
    for t in range(T):
        for s in range(idx.shape[1]):
            e = int(idx[t, s])
            if e not in covered and (row_of is None or row_of[t, s] >= 0):
                covered.add(e)
                chosen.add(t)
        if len(covered) == E:
            break
    return np.array(sorted(chosen), np.int32)


def check_routing(idx, gate, ref):
    """Selected experts bit-exact per token; slot order equal to the oracle's
    except between choices whose oracle keys tie within TIE_KEY; gates
    compared expert by expert.  Returns the number of tokens whose slot order
    differs (all within ties)."""
    idx = np.asarray(idx)
    gate = np.asarray(gate, np.float64)
    ridx, rgate, rkey = ref["idx"], ref["gate"], ref["sel_key"]
    np.testing.assert_array_equal(np.sort(idx, 1), np.sort(ridx, 1))
    swapped = np.nonzero((idx != ridx).any(1))[0]
    for t in swapped:
        key_of = dict(zip(ridx[t].tolist(), rkey[t].tolist()))
        keys = np.array([key_of[e] for e in idx[t].tolist()])
        assert np.all(np.diff(keys) <= TIE_KEY), "token %d: slot order is not a valid tie order" % t
    oi = np.argsort(idx, 1, kind="stable")
    ro = np.argsort(ridx, 1, kind="stable")
    g_sorted = np.take_along_axis(gate, oi, 1)
    r_sorted = np.take_along_axis(rgate, ro, 1)
    assert np.max(np.abs(g_sorted - r_sorted), initial=0.0) <= TOL_GATE
    return len(swapped)
