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


# ---------------------------------------------------------------- FP8 experts
# The same layer with FP8 (e4m3) experts, written from the format's bit
# fields and a nearest-value search over the whole code table (no shared
# code with the C oracle's closed-form rounding).

def _e4m3_table():
    """Value of every e4m3 code 0..255 from its sign / exponent / mantissa."""
    c = np.arange(256)
    s, e, m = c >> 7, (c >> 3) & 15, c & 7
    mag = np.where(e == 0, m / 8.0 * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where(s == 1, -mag, mag)
    val[(e == 15) & (m == 7)] = np.nan
    return val


E4M3 = _e4m3_table()


def e4m3_nearest(q):
    """Code of the e4m3 value nearest to each float32 q, by searching the
    table of the 127 finite magnitudes; ties go to the even code; the sign
    bit follows q's sign (so a negative q that rounds to zero gives -0)."""
    q = np.asarray(q, np.float32)
    a = np.abs(q.astype(np.float64)).ravel()
    mags = E4M3[:127]                                 # codes 0x00 .. 0x7E, increasing
    dist = np.abs(a[:, None] - mags[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    # among equally near codes prefer the even one (at most two candidates)
    even = cand & (np.arange(127)[None, :] % 2 == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    code = pick.astype(np.uint8) | np.where(np.signbit(q.ravel()), 0x80, 0).astype(np.uint8)
    return code.reshape(q.shape)


def bf16_round(h):
    """Nearest bf16 (ties to even) of float64 values, returned as float64:
    keep the top 7 fraction bits of the float64 pattern."""
    h = np.asarray(h, np.float64)
    bits = h.view(np.uint64)
    drop = np.uint64(52 - 7)
    lsb = (bits >> drop) & np.uint64(1)
    rounded = (bits + (np.uint64(1) << (drop - np.uint64(1))) - np.uint64(1) + lsb) >> drop << drop
    out = rounded.view(np.float64)
    return np.where(h == 0, h, out)


def quantize_rows_np(v):
    """Per-row e4m3 quantization in float32 arithmetic: inv = 448 / amax,
    code = nearest(v * inv), scale = amax / 448."""
    v = np.asarray(v, np.float32)
    amax = np.abs(v).max(axis=1)
    with np.errstate(divide="ignore"):
        inv = np.where(amax > 0, np.float32(448.0) / amax, np.float32(0.0)).astype(np.float32)
    codes = e4m3_nearest((v * inv[:, None]).astype(np.float32))
    scale = (amax / np.float32(448.0)).astype(np.float32)
    return codes, scale


def dequant_rows(codes, scale):
    return E4M3[np.asarray(codes, np.uint8)] * np.asarray(scale, np.float64)[..., None]


def expert_fn_fp8(act, xd, Wa, Wb, Wo, b_a=None, b_o=None):
    """One FP8 expert on dequantized rows xd; Wa/Wb/Wo dequantized weights.
    H is rounded to bf16 and quantized per row before the second product."""
    a = xd @ Wa.T
    if act == "gelu":
        if b_a is not None:
            a = a + b_a
        h = a * stats.norm.cdf(a)
    else:
        h = a * special.expit(a) * (xd @ Wb.T)
    hc, hs = quantize_rows_np(bf16_round(h).astype(np.float32))
    o = dequant_rows(hc, hs) @ Wo.T
    if b_o is not None:
        o = o + b_o
    return o


def layer_fp8(x, Wr, weights, k, *, act, score="softmax", renorm=1, capacity=-1,
              logit_bias=None, sel_bias=None):
    """The layer with FP8 experts.  weights: e4m3 codes W1, Wu, W2 (Wsg, Wsu,
    Wsd) with per-output-channel scales "<name>_scale", biases b1, b2.
    Returns dict(y, idx, gate, x8, xs)."""
    idx, gate, _, _ = route(x, Wr, k, score=score, renorm=renorm, logit_bias=logit_bias, sel_bias=sel_bias)
    x8, xs = quantize_rows_np(_f64(x).astype(np.float32))
    xd = dequant_rows(x8, xs)
    T, d = xd.shape
    E = np.asarray(Wr).shape[1]

    def wdeq(name):
        if weights.get(name) is None:
            return None
        return E4M3[np.asarray(weights[name], np.uint8)] * np.asarray(weights[name + "_scale"], np.float64)[..., None]

    W1, Wu, W2 = wdeq("W1"), wdeq("Wu"), wdeq("W2")
    b1 = np.asarray(weights["b1"], np.float64) if weights.get("b1") is not None else None
    b2 = np.asarray(weights["b2"], np.float64) if weights.get("b2") is not None else None
    y = np.zeros((T, d), np.float64)
    for e in range(E):
        tok, slot = np.nonzero(idx == e)
        if capacity >= 0:
            tok, slot = tok[:capacity], slot[:capacity]
        if len(tok) == 0:
            continue
        o = expert_fn_fp8(act, xd[tok], W1[e], None if Wu is None else Wu[e], W2[e],
                          None if b1 is None else b1[e], None if b2 is None else b2[e])
        np.add.at(y, tok, o * gate[tok, slot][:, None])
    if weights.get("Wsg") is not None:
        y += expert_fn_fp8(act, xd, wdeq("Wsg"), wdeq("Wsu"), wdeq("Wsd"))
    return dict(y=y, idx=idx, gate=gate, x8=x8, xs=xs)


# ---------------------------------------------------------------- MX experts
# The same layer with block-scaled (MX) e4m3 experts: 32-value blocks along the
# contraction dimension share a power-of-two scale, found here by comparing the
# block maximum against every power of two (no shared code with the C
# oracle's frexp-based exponent) and applied to the table search above.

def quantize_mx_np(v):
    """(codes [rows, cols], scale bytes [rows, cols/32]) of a float32 matrix:
    X is the largest integer in [-127, 127] with 2^(X + 8) <= amax (-127 when
    no power qualifies or amax = 0); codes are the nearest e4m3 values of v / 2^X."""
    v = np.asarray(v, np.float32)
    rows, cols = v.shape
    blk = v.reshape(rows, cols // 32, 32).astype(np.float64)
    amax = np.abs(blk).max(axis=2)
    X = np.full(amax.shape, -127, np.int64)
    for e in range(-127, 128):
        X = np.where(amax >= 2.0 ** (e + 8), e, X)
    q = (blk / np.exp2(X.astype(np.float64))[..., None]).astype(np.float32)
    codes = e4m3_nearest(q).reshape(rows, cols)
    return codes, (X + 127).astype(np.uint8)


def dequant_mx(codes, scales):
    codes = np.asarray(codes, np.uint8)
    sc = np.repeat(np.asarray(scales, np.float64) - 127.0, 32, axis=-1)
    return E4M3[codes] * np.exp2(sc)


def expert_fn_mx(act, xd, Wa, Wb, Wo, b_a=None, b_o=None):
    """One MX expert on dequantized rows xd with dequantized weights; H is
    rounded to bf16 and MX-quantized along d_ff before the second product."""
    a = xd @ Wa.T
    if act == "gelu":
        if b_a is not None:
            a = a + b_a
        h = a * stats.norm.cdf(a)
    else:
        h = a * special.expit(a) * (xd @ Wb.T)
    hc, hs = quantize_mx_np(bf16_round(h).astype(np.float32))
    o = dequant_mx(hc, hs) @ Wo.T
    if b_o is not None:
        o = o + b_o
    return o


def layer_mx(x, Wr, weights, k, *, act, score="softmax", renorm=1, capacity=-1,
             logit_bias=None, sel_bias=None):
    """The layer with MX experts.  weights: e4m3 codes W1, Wu, W2 (Wsg, Wsu,
    Wsd) with scale bytes "<name>_scale" [..., out, in/32], biases b1, b2.
    Returns dict(y, idx, gate, x8, xs)."""
    idx, gate, _, _ = route(x, Wr, k, score=score, renorm=renorm, logit_bias=logit_bias, sel_bias=sel_bias)
    x8, xs = quantize_mx_np(_f64(x).astype(np.float32))
    xd = dequant_mx(x8, xs)
    T, d = xd.shape
    E = np.asarray(Wr).shape[1]

    def wdeq(name):
        if weights.get(name) is None:
            return None
        return dequant_mx(weights[name], weights[name + "_scale"])

    W1, Wu, W2 = wdeq("W1"), wdeq("Wu"), wdeq("W2")
    b1 = np.asarray(weights["b1"], np.float64) if weights.get("b1") is not None else None
    b2 = np.asarray(weights["b2"], np.float64) if weights.get("b2") is not None else None
    y = np.zeros((T, d), np.float64)
    for e in range(E):
        tok, slot = np.nonzero(idx == e)
        if capacity >= 0:
            tok, slot = tok[:capacity], slot[:capacity]
        if len(tok) == 0:
            continue
        o = expert_fn_mx(act, xd[tok], W1[e], None if Wu is None else Wu[e], W2[e],
                         None if b1 is None else b1[e], None if b2 is None else b2[e])
        np.add.at(y, tok, o * gate[tok, slot][:, None])
    if weights.get("Wsg") is not None:
        y += expert_fn_mx(act, xd, wdeq("Wsg"), wdeq("Wsu"), wdeq("Wsd"))
    return dict(y=y, idx=idx, gate=gate, x8=x8, xs=xs)


# ---------------------------------------------------------------- INT4 weight-only experts
# The layer with INT4 weight-only experts: nibbles unpacked with numpy bit
# operations, each weight rounded to bf16 from q * s, then the bf16 layer's
# dense expert on the dequantized matrices.

def w4_dequant_np(codes, scales):
    codes = np.asarray(codes, np.uint8)
    lo = (codes & 15).astype(np.int64) - 8
    hi = (codes >> 4).astype(np.int64) - 8
    q = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    s = np.repeat(_f64(np.asarray(scales, np.uint16)), 128, axis=-1)
    return bf16_round(q.astype(np.float64) * s)


def layer_w4(x, Wr, weights, k, *, act, score="softmax", renorm=1, capacity=-1, logit_bias=None, sel_bias=None):
    """The layer with INT4 weight-only experts (weights: packed codes W1, Wu,
    W2 (Wsg, Wsu, Wsd) with bf16-bit scales "<name>_scale", biases b1, b2)."""
    dq = {}
    for name in ("W1", "Wu", "W2", "Wsg", "Wsu", "Wsd"):
        if weights.get(name) is not None:
            dq[name] = w4_dequant_np(weights[name], weights[name + "_scale"])
    for name in ("b1", "b2"):
        if weights.get(name) is not None:
            dq[name] = np.asarray(weights[name], np.float64)
    return layer(x, Wr, dq, k, act=act, score=score, renorm=renorm, capacity=capacity, logit_bias=logit_bias,
                 sel_bias=sel_bias)
