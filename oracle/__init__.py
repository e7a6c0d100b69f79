"""CPU oracle for the MoE FFN layer forward pass -- TEST INFRASTRUCTURE ONLY.

Only the test-suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The CUDA library shares no code with it.

The arithmetic lives in ``moe_oracle.c`` (IEEE double, plain loops; every
function cites the page passage it writes out).  This module only marshals
numpy arrays in and out.  ``loop_over_experts`` holds a second, independent
formulation used to pin the first.

Inputs: x and expert weights are fp32 arrays or bf16 arrays given as their raw
uint16 bit patterns; router weights and biases are fp32.

Parity pins (tests/test_oracle_pins.py): brute-force top-k on tiny inputs,
library softmax / sigmoid for the gates, sums of counts, closed-form balance
loss (exactly 1 under uniform routing, E under collapse), the dense-FFN
special case (E = 1, k = 1) against a direct matrix product with library
GELU / SiLU, the full soft mixture (k = E, no renormalisation), and agreement
with the loop-over-experts formulation.
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
                     "oracle_routing_health"):
            getattr(lib, name).restype = ctypes.c_int
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
