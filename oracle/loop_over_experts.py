"""Second, independent CPU formulation of the MoE layer -- TEST INFRASTRUCTURE.

Written from the loop-over-experts description in "Fine-tuning and serving
MoE models" (intellisensei tutorial, "How an MoE layer actually works"): for
every expert, find the (token, slot) pairs that chose it, run the expert once
on those rows as one matrix product, scale by the gates and add the result
back into token order.  Routing follows the DynamicBiasMoERouter description
in "Fine-Tuning Mixture of Experts (MoE) Models: Router Optimization
Techniques" ("How It Works" 2): select on the (optionally biased) score, then
take gates from the unbiased scores of the selected experts.

It uses numpy / scipy library routines (matmul, softmax, expit, the normal
CDF) and shares no code with ``moe_oracle.c``; the two must agree to rounding.
For small shapes only (everything is dense fp64 in memory).
"""
import numpy as np
from scipy import special, stats


def _f64(a):
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def route(x, Wr, k, *, score="softmax", renorm=1, logit_bias=None, sel_bias=None):
    x = _f64(x)
    logits = x @ np.asarray(Wr, np.float64)
    if logit_bias is not None:
        logits = logits + np.asarray(logit_bias, np.float64)[None, :]
    if score == "softmax":
        probs = special.softmax(logits, axis=-1)
        key = logits.copy()
    else:
        sig = special.expit(logits)
        probs = sig / sig.sum(-1, keepdims=True)
        key = sig.copy()
    if sel_bias is not None:
        key = key + np.asarray(sel_bias, np.float64)[None, :]
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    for t in range(T):
        # stable sort on -key keeps the lower expert index first among equals
        idx[t] = np.argsort(-key[t], kind="stable")[:k]
    if score == "softmax":
        sel_logits = np.take_along_axis(logits, idx, axis=1)
        if renorm:
            gate = special.softmax(sel_logits, axis=-1)
        else:
            gate = np.take_along_axis(probs, idx, axis=1)
    else:
        s = np.take_along_axis(special.expit(logits), idx, axis=1)
        gate = s / s.sum(-1, keepdims=True)
    return idx, gate, probs, logits


def expert_fn(act, xs, W_a, W_b, W_o, b_a=None, b_o=None):
    """One expert on a batch of rows (nn.Linear [out,in] weights)."""
    if act == "gelu":
        a = xs @ W_a.T
        if b_a is not None:
            a = a + b_a
        h = a * stats.norm.cdf(a)
        o = h @ W_o.T
        if b_o is not None:
            o = o + b_o
        return o
    g = xs @ W_a.T
    u = xs @ W_b.T
    return (g * special.expit(g) * u) @ W_o.T


def layer(x, Wr, weights, k, *, act, score="softmax", renorm=1, capacity=-1,
          logit_bias=None, sel_bias=None):
    """Returns dict(y, idx, gate, counts, kept, perm_rows, f, P, loss)."""
    xf = _f64(x)
    T, d = xf.shape
    E = np.asarray(Wr).shape[1]
    idx, gate, probs, logits = route(x, Wr, k, score=score, renorm=renorm,
                                     logit_bias=logit_bias, sel_bias=sel_bias)
    W1 = _f64(weights["W1"])
    W2 = _f64(weights["W2"])
    Wu = _f64(weights["Wu"]) if weights.get("Wu") is not None else None
    b1 = np.asarray(weights["b1"], np.float64) if weights.get("b1") is not None else None
    b2 = np.asarray(weights["b2"], np.float64) if weights.get("b2") is not None else None
    y = np.zeros((T, d), np.float64)
    perm_rows = []          # (expert, token) of every kept assignment, in row order
    kept = np.zeros(E, np.int64)
    for e in range(E):
        tok, slot = np.nonzero(idx == e)      # row-major: ascending token
        if capacity >= 0:
            tok, slot = tok[:capacity], slot[:capacity]
        kept[e] = len(tok)
        if len(tok) == 0:
            continue
        perm_rows.extend((e, int(t)) for t in tok)
        o = expert_fn(act, xf[tok], W1[e], None if Wu is None else Wu[e], W2[e],
                      None if b1 is None else b1[e], None if b2 is None else b2[e])
        np.add.at(y, tok, o * gate[tok, slot][:, None])
    if weights.get("Wsg") is not None:
        Wsu = _f64(weights["Wsu"]) if weights.get("Wsu") is not None else None
        y += expert_fn(act, xf, _f64(weights["Wsg"]), Wsu, _f64(weights["Wsd"]))
    counts = np.bincount(idx.reshape(-1), minlength=E)
    f = counts / float(T * k)
    P = probs.mean(0)
    return dict(y=y, idx=idx, gate=gate, counts=counts, kept=kept, perm_rows=perm_rows,
                f=f, P=P, loss=float(E * np.sum(f * P)), logits=logits, probs=probs)
