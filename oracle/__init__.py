"""CPU oracle for the MoE FFN layer forward pass -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (IEEE double, plain loops; every
function cites the page passage it writes out).  This module only marshals
numpy arrays in and out.  ``loop_over_experts`` holds a second, independent
formulation used to pin the first.

Inputs: x and expert weights are fp32 arrays or bf16 arrays given as their raw
uint16 bit patterns; router weights and biases are fp32.

FP8 experts (``e4m3_value``, ``e4m3_round``, ``quantize_rows``,
``expert_apply_fp8``, ``layer_tokens_fp8``): e4m3 codes with per-channel
weight scales and per-row activation scales, defined in ``moe_oracle.c``.
Block-scaled (MX) FP8 experts (``quantize_mx``, ``mx_value``,
``expert_apply_mx``, ``layer_tokens_mx``): e4m3 codes with one power-of-two
(E8M0) scale per 32 values along the contraction dimension.  INT4
weight-only experts (``w4_dequant``, ``expert_apply_w4``, ``layer_tokens_w4``):
signed 4-bit weights, two per byte, one bf16 scale per 128 inputs of a row,
bf16 activations.

Parity pins (tests/test_oracle_pins.py): brute-force top-k on tiny inputs,
library softmax / sigmoid for the gates, sums of counts, closed-form balance
loss (exactly 1 under uniform routing, E under collapse), the dense-FFN
special case (E = 1, k = 1) against a direct matrix product with library
GELU / SiLU, the full soft mixture (k = E, no renormalisation), and agreement
with the loop-over-experts formulation.  FP8: every e4m3 code's value and the
rounding of fp32 values against the library's float8_e4m3fn type and a brute-
force nearest-code search, the row quantizer's closed facts (largest code 448,
error within half a step, zero rows), and the FP8 experts against an
independent loop-over-experts formulation.
"""
import ctypes
import os

import numpy as np

from . import build as _build

I32P = ctypes.POINTER(ctypes.c_int32)
F64P = ctypes.POINTER(ctypes.c_double)


class Dims(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int32) for n in (
        "T", "d", "E", "d_ff", "k", "xw_dtype", "act", "score", "renorm",
        "capacity", "d_ff_shared", "nthreads")]


_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        lib.oracle_capacity.restype = ctypes.c_int32
        lib.oracle_capacity.argtypes = [ctypes.c_double, ctypes.c_int32, ctypes.c_int32, ctypes.c_int32]
        for name in ("oracle_route", "oracle_dispatch", "oracle_balance",
                     "oracle_expert_apply", "oracle_layer_tokens", "oracle_bias_update",
                     "oracle_routing_health", "oracle_quantize_rows", "oracle_expert_apply_fp8",
                     "oracle_layer_backward", "oracle_quantize_mx", "oracle_expert_apply_mx",
                     "oracle_expert_apply_w4", "oracle_w4_dequant"):
            getattr(lib, name).restype = ctypes.c_int
        lib.oracle_e4m3_value.restype = ctypes.c_double
        lib.oracle_e4m3_value.argtypes = [ctypes.c_uint8]
        lib.oracle_e4m3_round.restype = ctypes.c_uint8
        lib.oracle_e4m3_round.argtypes = [ctypes.c_float]
        _lib = lib
    return _lib


def default_threads() -> int:
    return max(1, len(os.sched_getaffinity(0)))


def _ptr(a):
    if a is None:
        return None
    return ctypes.c_void_p(a.ctypes.data)


def _raw(a, what):
    """x / expert weights: fp32 array or bf16 bit patterns (uint16)."""
    if a is None:
        return None
    a = np.ascontiguousarray(a)
    if a.dtype not in (np.float32, np.uint16):
        raise TypeError("%s must be float32 or uint16 (bf16 bits), got %s" % (what, a.dtype))
    return a


def _f32(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float32)


def capacity(capacity_factor: float, k: int, T: int, E: int) -> int:
    """Per-expert capacity floor(c*k*T/E); -1 for no limit (c <= 0)."""
    return int(_load().oracle_capacity(float(capacity_factor), int(k), int(T), int(E)))


def make_dims(T, d, E, d_ff, k, *, x_dtype, act="swiglu", score="softmax", renorm=1,
              capacity=-1, d_ff_shared=0, nthreads=None):
    return Dims(T=T, d=d, E=E, d_ff=d_ff, k=k,
                xw_dtype={"f32": 0, "bf16": 1}[x_dtype],
                act={"gelu": 0, "swiglu": 1}[act],
                score={"softmax": 0, "sigmoid": 1}[score],
                renorm=int(renorm), capacity=int(capacity), d_ff_shared=int(d_ff_shared),
                nthreads=int(nthreads or default_threads()))


def route(dims, x, Wr, logit_bias=None, sel_bias=None, tokens=None, want_logits=False,
          want_pnorm=True):
    """Router + selection + gates for all tokens (or the listed ones).

    Returns dict(idx [n,k] int32, gate [n,k] f64, margin [n] f64,
    sel_key [n,k] f64 (selection key of each choice), pnorm [n,E] f64
    (optional), logits [n,E] f64 (optional))."""
    lib = _load()
    x = _raw(x, "x")
    Wr = _f32(Wr)
    lb, sb = _f32(logit_bias), _f32(sel_bias)
    tok = None if tokens is None else np.ascontiguousarray(tokens, dtype=np.int32)
    n = dims.T if tok is None else len(tok)
    out = dict(idx=np.empty((n, dims.k), np.int32), gate=np.empty((n, dims.k), np.float64),
               margin=np.empty(n, np.float64), sel_key=np.empty((n, dims.k), np.float64))
    if want_pnorm:
        out["pnorm"] = np.empty((n, dims.E), np.float64)
    if want_logits:
        out["logits"] = np.empty((n, dims.E), np.float64)
    rc = lib.oracle_route(ctypes.byref(dims), ctypes.c_int64(n), _ptr(tok), _ptr(x), _ptr(Wr),
                          _ptr(lb), _ptr(sb), _ptr(out["idx"]), _ptr(out["gate"]),
                          _ptr(out.get("logits")), _ptr(out.get("pnorm")), _ptr(out["margin"]),
                          _ptr(out["sel_key"]))
    if rc:
        raise ValueError("oracle_route rejected its arguments")
    return out


def dispatch(dims, idx):
    """Counts, capacity, offsets and the (expert, token)-ordered permutation."""
    lib = _load()
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    E, T, k = dims.E, dims.T, dims.k
    out = dict(counts=np.empty(E, np.int32), kept=np.empty(E, np.int32),
               offsets=np.empty(E + 1, np.int32), row_of=np.empty((T, k), np.int32),
               row_token=np.full(max(T * k, 1), -1, np.int32))
    nd = ctypes.c_int32(0)
    rc = lib.oracle_dispatch(ctypes.byref(dims), _ptr(idx), _ptr(out["counts"]), _ptr(out["kept"]),
                             _ptr(out["offsets"]), _ptr(out["row_of"]), _ptr(out["row_token"]),
                             ctypes.byref(nd))
    if rc:
        raise ValueError("oracle_dispatch: expert index out of range")
    out["n_dropped"] = int(nd.value)
    out["row_token"] = out["row_token"][: int(out["offsets"][E])]
    return out


def balance(dims, counts, pnorm):
    """f, P and the balance loss L = E * sum f P (all fp64)."""
    lib = _load()
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    pnorm = np.ascontiguousarray(pnorm, dtype=np.float64)
    assert pnorm.shape == (dims.T, dims.E)
    f = np.empty(dims.E, np.float64)
    P = np.empty(dims.E, np.float64)
    L = ctypes.c_double(0.0)
    lib.oracle_balance(ctypes.byref(dims), _ptr(counts), _ptr(pnorm), _ptr(f), _ptr(P), ctypes.byref(L))
    return dict(f=f, P=P, loss=float(L.value))


def _weights(w):
    return (_raw(w.get("W1"), "W1"), _f32(w.get("b1")), _raw(w.get("Wu"), "Wu"),
            _raw(w.get("W2"), "W2"), _f32(w.get("b2")), _raw(w.get("Wsg"), "Wsg"),
            _raw(w.get("Wsu"), "Wsu"), _raw(w.get("Wsd"), "Wsd"))


def expert_apply(dims, x, weights, token, expert, scale=None):
    """out[r] = scale[r] * E_{expert[r]}(x[token[r]]); expert == E is the shared expert.

    weights: dict with W1 (GELU W1 / SwiGLU W_gate) [E,d_ff,d], b1 [E,d_ff],
    Wu (SwiGLU W_up) [E,d_ff,d], W2 (W_down) [E,d,d_ff], b2 [E,d],
    Wsg/Wsu/Wsd for the shared expert."""
    lib = _load()
    x = _raw(x, "x")
    token = np.ascontiguousarray(token, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float64)
    out = np.empty((len(token), dims.d), np.float64)
    ws = _weights(weights)
    rc = lib.oracle_expert_apply(ctypes.byref(dims), ctypes.c_int64(len(token)), _ptr(token), _ptr(expert),
                                 _ptr(sc), _ptr(x), *[_ptr(a) for a in ws], _ptr(out))
    if rc:
        raise ValueError("oracle_expert_apply: bad expert id")
    return out


def layer_tokens(dims, x, weights, idx, gate, row_of, tokens):
    """y[n] for the listed tokens: gate-weighted sum of kept experts (+ shared)."""
    lib = _load()
    x = _raw(x, "x")
    tokens = np.ascontiguousarray(tokens, dtype=np.int32)
    idx = np.ascontiguousarray(idx, dtype=np.int32)
    gate = np.ascontiguousarray(gate, dtype=np.float64)
    ro = None if row_of is None else np.ascontiguousarray(row_of, dtype=np.int32)
    y = np.empty((len(tokens), dims.d), np.float64)
    ws = _weights(weights)
    lib.oracle_layer_tokens(ctypes.byref(dims), ctypes.c_int64(len(tokens)), _ptr(tokens), _ptr(x),
                            _ptr(idx), _ptr(gate), _ptr(ro), *[_ptr(a) for a in ws], _ptr(y))
    return y


def forward(dims, x, Wr, weights, logit_bias=None, sel_bias=None, tokens=None):
    """Whole layer: routing/dispatch/balance over all T, outputs for `tokens`
    (all tokens when None)."""
    r = route(dims, x, Wr, logit_bias, sel_bias)
    dp = dispatch(dims, r["idx"])
    bal = balance(dims, dp["counts"], r["pnorm"])
    tok = np.arange(dims.T, dtype=np.int32) if tokens is None else np.asarray(tokens, np.int32)
    y = layer_tokens(dims, x, weights, r["idx"], r["gate"], dp["row_of"], tok)
    out = dict(r)
    out.update(dp)
    out.update(bal)
    out["y"] = y
    out["tokens"] = tok
    return out


def layer_backward(dims, x, Wr, weights, dy, alpha=0.0, logit_bias=None, sel_bias=None):
    """Gradient of sum_t <dy_t, y_t> + alpha * L_aux (all fp64): dict with dx
    [T,d], dWr [d,E], dbeta [E] (the logit offset), dW1, db1, dWu, dW2, db2,
    dWsg, dWsu, dWsd (the shapes of the weights; absent weights give None)."""
    lib = _load()
    x = _raw(x, "x")
    Wr = _f32(Wr)
    lb, sb = _f32(logit_bias), _f32(sel_bias)
    dy = np.ascontiguousarray(dy, dtype=np.float64)
    T, d, E, F, S = dims.T, dims.d, dims.E, dims.d_ff, dims.d_ff_shared
    assert dy.shape == (T, d)
    out = dict(dx=np.empty((T, d)), dWr=np.empty((d, E)), dbeta=np.empty(E))
    present = {k for k, v in weights.items() if v is not None}
    shapes = dict(dW1=("W1", (E, F, d)), db1=("b1", (E, F)), dWu=("Wu", (E, F, d)), dW2=("W2", (E, d, F)),
                  db2=("b2", (E, d)), dWsg=("Wsg", (S, d)), dWsu=("Wsu", (S, d)), dWsd=("Wsd", (d, S)))
    for name, (src, shp) in shapes.items():
        out[name] = np.empty(shp) if src in present else None
    ws = _weights(weights)
    rc = lib.oracle_layer_backward(ctypes.byref(dims), _ptr(x), _ptr(Wr), _ptr(lb), _ptr(sb), *[_ptr(a) for a in ws],
                                   _ptr(dy), ctypes.c_double(alpha), _ptr(out["dx"]), _ptr(out["dWr"]),
                                   _ptr(out["dbeta"]), *[_ptr(out[n]) for n in shapes])
    if rc:
        raise ValueError("oracle_layer_backward rejected its arguments")
    return out


def bias_update(dims, counts, bias, gamma):
    """b_e - gamma * sign(count_e - T k / E), returned as a new float32 array."""
    lib = _load()
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    b = np.array(bias, dtype=np.float32, copy=True)
    lib.oracle_bias_update(ctypes.byref(dims), _ptr(counts), ctypes.c_double(gamma), _ptr(b))
    return b


def routing_health(dims, counts, P):
    """dict(entropy = -sum P log P, ratio = max/min count, max_share)."""
    lib = _load()
    counts = np.ascontiguousarray(counts, dtype=np.int32)
    P = np.ascontiguousarray(P, dtype=np.float64)
    out = np.empty(3, np.float64)
    lib.oracle_routing_health(ctypes.byref(dims), _ptr(counts), _ptr(P), _ptr(out))
    return dict(entropy=float(out[0]), ratio=float(out[1]), max_share=float(out[2]))


def bf16_bits_to_f64(a):
    """Exact widening of bf16 bit patterns (uint16) to float64."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


# ---------------------------------------------------------------- FP8 experts
def e4m3_value(codes):
    """float64 value of each e4m3 code (NaN for the NaN codes)."""
    lib = _load()
    c = np.asarray(codes, dtype=np.uint8)
    return np.array([lib.oracle_e4m3_value(int(v)) for v in c.ravel()], np.float64).reshape(c.shape)


def e4m3_round(q):
    """e4m3 code nearest to each fp32 value (ties to even, saturating at 448)."""
    lib = _load()
    q = np.asarray(q, dtype=np.float32)
    return np.array([lib.oracle_e4m3_round(float(v)) for v in q.ravel()], np.uint8).reshape(q.shape)


def quantize_rows(v):
    """(codes uint8 [rows, cols], scale float32 [rows]) of a float32 matrix."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    codes = np.empty((rows, cols), np.uint8)
    scale = np.empty(rows, np.float32)
    lib.oracle_quantize_rows(_ptr(v), ctypes.c_int64(rows), ctypes.c_int32(cols), ctypes.c_int64(cols),
                             _ptr(codes), _ptr(scale))
    return codes, scale


def quantize_mx(v):
    """MX quantization of a float32 matrix (columns a multiple of 32): (codes
    uint8 [rows, cols], scale bytes uint8 [rows, cols / 32], E8M0: 2^(s - 127))."""
    lib = _load()
    v = np.ascontiguousarray(v, dtype=np.float32)
    rows, cols = v.shape
    codes = np.empty((rows, cols), np.uint8)
    scales = np.empty((rows, cols // 32), np.uint8)
    if lib.oracle_quantize_mx(_ptr(v), ctypes.c_int64(rows), ctypes.c_int32(cols), ctypes.c_int64(cols),
                              _ptr(codes), _ptr(scales)):
        raise ValueError("quantize_mx: columns must be a positive multiple of 32")
    return codes, scales


def mx_value(codes, scales):
    """float64 values of MX codes with their block scale bytes (last axis of
    codes = 32 x last axis of scales)."""
    codes = np.asarray(codes, np.uint8)
    sc = np.repeat(np.asarray(scales, np.int64), 32, axis=-1)
    return np.ldexp(e4m3_value(codes.ravel()).reshape(codes.shape), (sc - 127).astype(np.int32))


def _mx_weights(w):
    def u8(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)
    return (u8(w.get("W1")), u8(w.get("W1_scale")), _f32(w.get("b1")),
            u8(w.get("Wu")), u8(w.get("Wu_scale")),
            u8(w.get("W2")), u8(w.get("W2_scale")), _f32(w.get("b2")),
            u8(w.get("Wsg")), u8(w.get("Wsg_scale")), u8(w.get("Wsu")), u8(w.get("Wsu_scale")),
            u8(w.get("Wsd")), u8(w.get("Wsd_scale")))


def expert_apply_mx(dims, x8, xs, weights, token, expert, scale=None):
    """out[r] = scale[r] * Emx_{expert[r]}(x8[token[r]]) with MX experts.

    x8: e4m3 codes [T, d] with scale bytes xs [T, d/32]; weights: W1, Wu, W2
    (and Wsg, Wsu, Wsd) as e4m3 codes with scale bytes "<name>_scale" of shape
    [..., out, in/32]; biases b1, b2 fp32."""
    lib = _load()
    x8 = np.ascontiguousarray(x8, dtype=np.uint8)
    xs = np.ascontiguousarray(xs, dtype=np.uint8)
    token = np.ascontiguousarray(token, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float64)
    out = np.empty((len(token), dims.d), np.float64)
    ws = _mx_weights(weights)
    rc = lib.oracle_expert_apply_mx(ctypes.byref(dims), ctypes.c_int64(len(token)), _ptr(token), _ptr(expert),
                                    _ptr(sc), _ptr(x8), _ptr(xs), *[_ptr(a) for a in ws], _ptr(out))
    if rc:
        raise ValueError("oracle_expert_apply_mx: bad expert id or dimension not a multiple of 32")
    return out


def layer_tokens_mx(dims, x8, xs, weights, idx, gate, row_of, tokens):
    """y[n] for the listed tokens with MX experts: the gate-weighted sum of
    the kept experts (+ the shared expert, weight 1), summed in float64."""
    idx = np.asarray(idx, np.int32)
    gate = np.asarray(gate, np.float64)
    tokens = np.asarray(tokens, np.int32)
    tok, ex, g, owner = [], [], [], []
    for n, t in enumerate(tokens):
        for s in range(dims.k):
            if row_of is not None and row_of[t, s] < 0:
                continue
            tok.append(t); ex.append(idx[t, s]); g.append(gate[t, s]); owner.append(n)
        if dims.d_ff_shared > 0:
            tok.append(t); ex.append(dims.E); g.append(1.0); owner.append(n)
    y = np.zeros((len(tokens), dims.d), np.float64)
    if tok:
        rows = expert_apply_mx(dims, x8, xs, weights, np.array(tok), np.array(ex), np.array(g))
        for r, n in enumerate(owner):
            y[n] += rows[r]
    return y


def w4_dequant(codes, scales):
    """float64 values of INT4 weights: codes uint8 [rows, cols/2] (low nibble
    = even input, nibble = q + 8), scales bf16 bits uint16 [rows, cols/128]."""
    lib = _load()
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    scales = np.ascontiguousarray(scales, dtype=np.uint16)
    rows, half = codes.shape
    out = np.empty((rows, half * 2), np.float64)
    if lib.oracle_w4_dequant(_ptr(codes), _ptr(scales), ctypes.c_int64(rows), ctypes.c_int32(half * 2), _ptr(out)):
        raise ValueError("w4_dequant: columns must be a positive multiple of 128")
    return out


def _w4_weights(w):
    def u8(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)

    def u16(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.uint16)
    return (u8(w.get("W1")), u16(w.get("W1_scale")), _f32(w.get("b1")),
            u8(w.get("Wu")), u16(w.get("Wu_scale")),
            u8(w.get("W2")), u16(w.get("W2_scale")), _f32(w.get("b2")),
            u8(w.get("Wsg")), u16(w.get("Wsg_scale")), u8(w.get("Wsu")), u16(w.get("Wsu_scale")),
            u8(w.get("Wsd")), u16(w.get("Wsd_scale")))


def expert_apply_w4(dims, x, weights, token, expert, scale=None):
    """out[r] = scale[r] * Ew4_{expert[r]}(x[token[r]]) with INT4 weight-only
    experts.  x: bf16 bits [T, d]; weights: W1, Wu, W2 (and Wsg, Wsu, Wsd) as
    packed codes [..., out, in/2] with bf16-bit scales "<name>_scale"
    [..., out, in/128]; biases b1, b2 fp32."""
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.uint16)
    token = np.ascontiguousarray(token, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float64)
    out = np.empty((len(token), dims.d), np.float64)
    ws = _w4_weights(weights)
    rc = lib.oracle_expert_apply_w4(ctypes.byref(dims), ctypes.c_int64(len(token)), _ptr(token), _ptr(expert),
                                    _ptr(sc), _ptr(x), *[_ptr(a) for a in ws], _ptr(out))
    if rc:
        raise ValueError("oracle_expert_apply_w4: bad expert id or dimension not a multiple of 128")
    return out


def layer_tokens_w4(dims, x, weights, idx, gate, row_of, tokens):
    """y[n] for the listed tokens with INT4 weight-only experts: the
    gate-weighted sum of the kept experts (+ the shared expert, weight 1)."""
    idx = np.asarray(idx, np.int32)
    gate = np.asarray(gate, np.float64)
    tokens = np.asarray(tokens, np.int32)
    tok, ex, g, owner = [], [], [], []
    for n, t in enumerate(tokens):
        for s in range(dims.k):
            if row_of is not None and row_of[t, s] < 0:
                continue
            tok.append(t); ex.append(idx[t, s]); g.append(gate[t, s]); owner.append(n)
        if dims.d_ff_shared > 0:
            tok.append(t); ex.append(dims.E); g.append(1.0); owner.append(n)
    y = np.zeros((len(tokens), dims.d), np.float64)
    if tok:
        rows = expert_apply_w4(dims, x, weights, np.array(tok), np.array(ex), np.array(g))
        for r, n in enumerate(owner):
            y[n] += rows[r]
    return y


def _fp8_weights(w):
    def u8(a):
        return None if a is None else np.ascontiguousarray(a, dtype=np.uint8)
    return (u8(w.get("W1")), _f32(w.get("W1_scale")), _f32(w.get("b1")),
            u8(w.get("Wu")), _f32(w.get("Wu_scale")),
            u8(w.get("W2")), _f32(w.get("W2_scale")), _f32(w.get("b2")),
            u8(w.get("Wsg")), _f32(w.get("Wsg_scale")), u8(w.get("Wsu")), _f32(w.get("Wsu_scale")),
            u8(w.get("Wsd")), _f32(w.get("Wsd_scale")))


def expert_apply_fp8(dims, x8, xs, weights, token, expert, scale=None):
    """out[r] = scale[r] * E8_{expert[r]}(x8[token[r]]) with FP8 experts.

    x8: e4m3 codes [T, d] with row scales xs [T]; weights: W1, Wu, W2 (and
    Wsg, Wsu, Wsd) as e4m3 codes with per-output-channel scales under the
    same names + "_scale", biases b1, b2 fp32."""
    lib = _load()
    x8 = np.ascontiguousarray(x8, dtype=np.uint8)
    xs = _f32(xs)
    token = np.ascontiguousarray(token, dtype=np.int32)
    expert = np.ascontiguousarray(expert, dtype=np.int32)
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.float64)
    out = np.empty((len(token), dims.d), np.float64)
    ws = _fp8_weights(weights)
    rc = lib.oracle_expert_apply_fp8(ctypes.byref(dims), ctypes.c_int64(len(token)), _ptr(token), _ptr(expert),
                                     _ptr(sc), _ptr(x8), _ptr(xs), *[_ptr(a) for a in ws], _ptr(out))
    if rc:
        raise ValueError("oracle_expert_apply_fp8: bad expert id")
    return out


def layer_tokens_fp8(dims, x8, xs, weights, idx, gate, row_of, tokens):
    """y[n] for the listed tokens with FP8 experts: the gate-weighted sum of
    the kept experts (+ the shared expert, weight 1), summed in float64."""
    idx = np.asarray(idx, np.int32)
    gate = np.asarray(gate, np.float64)
    tokens = np.asarray(tokens, np.int32)
    k = dims.k
    tok, ex, g, owner = [], [], [], []
    for n, t in enumerate(tokens):
        for s in range(k):
            if row_of is not None and row_of[t, s] < 0:
                continue
            tok.append(t); ex.append(idx[t, s]); g.append(gate[t, s]); owner.append(n)
        if dims.d_ff_shared > 0:
            tok.append(t); ex.append(dims.E); g.append(1.0); owner.append(n)
    y = np.zeros((len(tokens), dims.d), np.float64)
    if tok:
        rows = expert_apply_fp8(dims, x8, xs, weights, np.array(tok), np.array(ex), np.array(g))
        for r, n in enumerate(owner):
            y[n] += rows[r]
    return y
