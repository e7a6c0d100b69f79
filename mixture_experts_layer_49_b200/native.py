"""Thin ctypes binding of libmoe (include/moe.h).

Argument marshalling only: every step of the layer runs in the CUDA library.
Functions keep the C names and take torch tensors that already live on the
GPU; they pass raw device pointers and the current CUDA stream through the
C ABI and raise MoEError on any non-OK status.  There is no fallback path:
if the library is missing or no GPU is present, calls fail.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

c_i32 = ctypes.c_int32
c_vp = ctypes.c_void_p

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_WORKSPACE, MOE_ERR_CUDA, \
    MOE_ERR_TIMEOUT, MOE_ERR_DEVICE_BOUNDS = range(7)
MOE_F32, MOE_BF16 = 0, 1
MOE_ACT_GELU_BIAS, MOE_ACT_SWIGLU = 0, 1
MOE_SCORE_SOFTMAX, MOE_SCORE_SIGMOID = 0, 1

EXPORTS = ("moe_workspace_size", "moe_capacity", "moe_router_blocks", "moe_perm_rows",
           "moe_workspace_init", "moe_router_topk", "moe_permute", "moe_grouped_ffn",
           "moe_combine", "moe_balance_stats", "moe_forward", "moe_get_device_status",
           "moe_status_string", "moe_last_error_detail", "moe_permute_noalloc",
           "moe_bias_update", "moe_routing_health", "moe_check_wait_timeout",
           "moe_quantize_rows_e4m3", "moe_grouped_ffn_fp8", "moe_forward_fp8", "moe_workspace_view",
           "moe_ep_workspace_size", "moe_ep_grouped_ffn", "moe_backward_workspace_size", "moe_backward",
           "moe_forward_train",
           "moe_quantize_rows_mx", "moe_grouped_ffn_mx_workspace_size", "moe_grouped_ffn_mx",
           "moe_router_freeze", "moe_forward_mx", "moe_grouped_ffn_w4", "moe_forward_w4")


class MoeFp8Experts(ctypes.Structure):
    """moe_fp8_experts: e4m3 expert weights (device pointers) and their
    per-output-channel fp32 scales."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "W1", "W1_scale", "Wu", "Wu_scale", "W2", "W2_scale",
        "Wsh_g", "Wsh_g_scale", "Wsh_u", "Wsh_u_scale", "Wsh_d", "Wsh_d_scale")]


class MoeMxExperts(ctypes.Structure):
    """moe_mx_experts: block-scaled e4m3 expert weights (device pointers),
    their E8M0 scale bytes and the scale row stride sld."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "W1", "W1_scale", "Wu", "Wu_scale", "W2", "W2_scale",
        "Wsh_g", "Wsh_g_scale", "Wsh_u", "Wsh_u_scale", "Wsh_d", "Wsh_d_scale")] + [("sld", ctypes.c_int32)]


class MoeW4Experts(ctypes.Structure):
    """moe_w4_experts: INT4 weight-only expert weights (packed codes), their
    bf16 group scales (as bytes) and the scale row stride sld."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "W1", "W1_scale", "Wu", "Wu_scale", "W2", "W2_scale",
        "Wsh_g", "Wsh_g_scale", "Wsh_u", "Wsh_u_scale", "Wsh_d", "Wsh_d_scale")] + [("sld", ctypes.c_int32)]


class MoeWsView(ctypes.Structure):
    """moe_ws_view: device addresses of the forward pass's intermediate
    results inside a workspace."""
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "kept", "offsets", "row_of", "row_token", "row_gate", "x_perm", "H", "y_perm")] + [
        ("h_stride", ctypes.c_int64)]


class MoEError(RuntimeError):
    def __init__(self, status, where, detail=""):
        self.status = status
        super().__init__("%s: %s (%d)%s" % (where, status_string(status), status,
                                            (" -- " + detail) if detail else ""))


class MoeConfig(ctypes.Structure):
    _fields_ = [("T", c_i32), ("d_model", c_i32), ("E", c_i32), ("d_ff", c_i32),
                ("top_k", c_i32), ("dtype", c_i32), ("act", c_i32), ("score", c_i32),
                ("renorm", c_i32), ("capacity_factor", ctypes.c_float), ("d_ff_shared", c_i32)]

    def __repr__(self):
        return "MoeConfig(%s)" % ", ".join("%s=%s" % (n, getattr(self, n)) for n, _ in self._fields_)


_lib = None


def lib():
    """Load libmoe.so (building it in-tree first if it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if not os.path.exists(path) or _build.stale():
            path = _build.build()
        L = ctypes.CDLL(path)
        P = ctypes.POINTER
        L.moe_workspace_size.restype = ctypes.c_size_t
        L.moe_workspace_size.argtypes = [P(MoeConfig)]
        for n in ("moe_capacity", "moe_router_blocks"):
            getattr(L, n).restype = c_i32
            getattr(L, n).argtypes = [P(MoeConfig)]
        L.moe_perm_rows.restype = ctypes.c_int64
        L.moe_perm_rows.argtypes = [P(MoeConfig)]
        L.moe_status_string.restype = ctypes.c_char_p
        L.moe_status_string.argtypes = [ctypes.c_int]
        L.moe_last_error_detail.restype = ctypes.c_char_p
        L.moe_last_error_detail.argtypes = []
        for n in ("moe_workspace_init", "moe_router_topk", "moe_permute", "moe_grouped_ffn",
                  "moe_combine", "moe_balance_stats", "moe_forward", "moe_get_device_status"):
            getattr(L, n).restype = ctypes.c_int
        L.moe_workspace_init.argtypes = [c_vp, ctypes.c_size_t, c_vp]
        L.moe_router_topk.argtypes = [P(MoeConfig)] + [c_vp] * 9 + [ctypes.c_size_t, c_vp]
        L.moe_permute.argtypes = [P(MoeConfig)] + [c_vp] * 12 + [ctypes.c_size_t, c_vp]
        L.moe_grouped_ffn.argtypes = [P(MoeConfig)] + [c_vp] * 14 + [ctypes.c_size_t, c_vp]
        L.moe_combine.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [ctypes.c_size_t, c_vp]
        L.moe_balance_stats.argtypes = [P(MoeConfig)] + [c_vp] * 6
        L.moe_forward.argtypes = [P(MoeConfig)] + [c_vp] * 22 + [ctypes.c_size_t, c_vp]
        L.moe_forward_train.restype = ctypes.c_int
        L.moe_forward_train.argtypes = [P(MoeConfig)] + [c_vp] * 22 + [ctypes.c_size_t, c_vp, ctypes.c_size_t, c_vp]
        L.moe_get_device_status.argtypes = [c_vp, c_vp, P(c_i32)]
        L.moe_bias_update.restype = ctypes.c_int
        L.moe_bias_update.argtypes = [P(MoeConfig), c_vp, c_vp, ctypes.c_float, c_vp]
        L.moe_routing_health.restype = ctypes.c_int
        L.moe_routing_health.argtypes = [P(MoeConfig), c_vp, c_vp, c_vp, c_vp]
        L.moe_ep_workspace_size.restype = ctypes.c_size_t
        L.moe_ep_workspace_size.argtypes = [P(MoeConfig), c_i32, ctypes.c_int64]
        L.moe_ep_grouped_ffn.restype = ctypes.c_int
        L.moe_ep_grouped_ffn.argtypes = [P(MoeConfig), c_i32, c_vp, ctypes.c_int64] + [c_vp] * 9 + [
            ctypes.c_size_t, c_vp]
        L.moe_backward_workspace_size.restype = ctypes.c_size_t
        L.moe_backward_workspace_size.argtypes = [P(MoeConfig)]
        L.moe_backward.restype = ctypes.c_int
        L.moe_backward.argtypes = [P(MoeConfig)] + [c_vp] * 15 + [ctypes.c_float] + [c_vp] * 11 + [
            c_vp, ctypes.c_size_t, c_vp, ctypes.c_size_t, c_vp]
        L.moe_workspace_view.restype = ctypes.c_int
        L.moe_workspace_view.argtypes = [P(MoeConfig), c_vp, ctypes.c_size_t, P(MoeWsView)]
        L.moe_check_wait_timeout.restype = ctypes.c_int
        L.moe_check_wait_timeout.argtypes = [c_vp, ctypes.c_uint64, c_vp]
        L.moe_permute_noalloc.restype = ctypes.c_int
        L.moe_permute_noalloc.argtypes = [P(MoeConfig)] + [c_vp] * 11 + [c_vp]
        L.moe_quantize_rows_e4m3.restype = ctypes.c_int
        L.moe_quantize_rows_e4m3.argtypes = [c_vp, ctypes.c_int64, c_i32, ctypes.c_int64, c_vp, ctypes.c_int64,
                                             c_vp, c_vp]
        L.moe_grouped_ffn_fp8.restype = ctypes.c_int
        L.moe_grouped_ffn_fp8.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [P(MoeFp8Experts)] + [c_vp] * 6 + [
            ctypes.c_size_t, c_vp]
        L.moe_router_freeze.restype = ctypes.c_int
        L.moe_router_freeze.argtypes = [P(MoeConfig), c_vp, c_vp, ctypes.c_size_t, c_vp]
        L.moe_grouped_ffn_w4.restype = ctypes.c_int
        L.moe_grouped_ffn_w4.argtypes = [P(MoeConfig)] + [c_vp] * 3 + [P(MoeW4Experts)] + [c_vp] * 5 + [
            ctypes.c_size_t, c_vp]
        L.moe_forward_w4.restype = ctypes.c_int
        L.moe_forward_w4.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [P(MoeW4Experts)] + [c_vp] * 12 + [
            ctypes.c_size_t, c_vp]
        L.moe_forward_mx.restype = ctypes.c_int
        L.moe_forward_mx.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [P(MoeMxExperts)] + [c_vp] * 12 + [
            ctypes.c_size_t, c_vp, ctypes.c_size_t, c_vp]
        L.moe_quantize_rows_mx.restype = ctypes.c_int
        L.moe_quantize_rows_mx.argtypes = [c_vp, ctypes.c_int64, c_i32, ctypes.c_int64, c_vp, ctypes.c_int64,
                                           c_vp, ctypes.c_int64, c_vp]
        L.moe_grouped_ffn_mx_workspace_size.restype = ctypes.c_size_t
        L.moe_grouped_ffn_mx_workspace_size.argtypes = [P(MoeConfig), c_i32]
        L.moe_grouped_ffn_mx.restype = ctypes.c_int
        L.moe_grouped_ffn_mx.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [P(MoeMxExperts)] + [c_vp] * 6 + [
            ctypes.c_size_t, c_vp]
        L.moe_forward_fp8.restype = ctypes.c_int
        L.moe_forward_fp8.argtypes = [P(MoeConfig)] + [c_vp] * 4 + [P(MoeFp8Experts)] + [c_vp] * 12 + [
            ctypes.c_size_t, c_vp]
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


def last_error_detail() -> str:
    return lib().moe_last_error_detail().decode()


def _check(rc, where):
    if rc != MOE_OK:
        raise MoEError(rc, where, last_error_detail())


def make_config(T, d_model, E, d_ff, top_k, *, dtype="bf16", act="swiglu", score="softmax",
                renorm=1, capacity_factor=0.0, d_ff_shared=0) -> MoeConfig:
    return MoeConfig(T=T, d_model=d_model, E=E, d_ff=d_ff, top_k=top_k,
                     dtype={"f32": MOE_F32, "bf16": MOE_BF16}[dtype],
                     act={"gelu": MOE_ACT_GELU_BIAS, "swiglu": MOE_ACT_SWIGLU}[act],
                     score={"softmax": MOE_SCORE_SOFTMAX, "sigmoid": MOE_SCORE_SIGMOID}[score],
                     renorm=int(renorm), capacity_factor=float(capacity_factor),
                     d_ff_shared=int(d_ff_shared))


def config_from_workload(wl, T=None) -> MoeConfig:
    return make_config(wl.T if T is None else T, wl.d_model, wl.E, wl.d_ff, wl.top_k,
                       dtype=wl.dtype, act=wl.act, score=wl.score, renorm=wl.renorm,
                       capacity_factor=wl.capacity_factor, d_ff_shared=wl.d_ff_shared)


def _p(t):
    """Device pointer of a CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError("expected a torch.Tensor")
    if not t.is_cuda:
        raise ValueError("libmoe takes device tensors; got one on %s" % t.device)
    if not t.is_contiguous():
        raise ValueError("libmoe takes contiguous tensors")
    return c_vp(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return c_vp(stream.cuda_stream)


def workspace_size(cfg) -> int:
    return int(lib().moe_workspace_size(ctypes.byref(cfg)))


def capacity(cfg) -> int:
    return int(lib().moe_capacity(ctypes.byref(cfg)))


def router_blocks(cfg) -> int:
    return int(lib().moe_router_blocks(ctypes.byref(cfg)))


def perm_rows(cfg) -> int:
    return int(lib().moe_perm_rows(ctypes.byref(cfg)))


def alloc_workspace(cfg, device="cuda", stream=None) -> torch.Tensor:
    n = workspace_size(cfg)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_workspace_size", last_error_detail())
    ws = torch.empty(n, dtype=torch.uint8, device=device)
    moe_workspace_init(ws, stream=stream)
    return ws


def moe_workspace_init(ws, stream=None):
    _check(lib().moe_workspace_init(_p(ws), ws.numel() * ws.element_size(), _stream(stream)),
           "moe_workspace_init")


def moe_router_topk(cfg, x, Wr, logit_bias, sel_bias, idx, gate, logits_out, psum, ws, stream=None):
    _check(lib().moe_router_topk(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias),
                                 _p(idx), _p(gate), _p(logits_out), _p(psum), _p(ws), ws.numel(),
                                 _stream(stream)), "moe_router_topk")


def moe_permute(cfg, x, idx, gate, counts, kept, offsets, row_of, row_token, row_gate, x_perm,
                n_dropped, ws, stream=None):
    _check(lib().moe_permute(ctypes.byref(cfg), _p(x), _p(idx), _p(gate), _p(counts), _p(kept),
                             _p(offsets), _p(row_of), _p(row_token), _p(row_gate), _p(x_perm),
                             _p(n_dropped), _p(ws), ws.numel(), _stream(stream)), "moe_permute")


def moe_permute_noalloc(cfg, x, idx, gate, counts, kept, offsets, row_of, row_token, row_gate, x_perm,
                        n_dropped, stream=None):
    """moe_permute without a workspace, for callers that cannot allocate
    device memory (scratch lives in a fixed array inside libmoe; calls that
    overlap on the GPU race on it; limit E * ceil(T/64) <= 262144)."""
    _check(lib().moe_permute_noalloc(ctypes.byref(cfg), _p(x), _p(idx), _p(gate), _p(counts), _p(kept),
                                     _p(offsets), _p(row_of), _p(row_token), _p(row_gate), _p(x_perm),
                                     _p(n_dropped), _stream(stream)), "moe_permute_noalloc")


def moe_grouped_ffn(cfg, x_perm, offsets, row_gate, W1, b1, Wu, W2, b2, x, Wsh_g, Wsh_u, Wsh_d,
                    y_perm, ws, stream=None):
    _check(lib().moe_grouped_ffn(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(row_gate), _p(W1),
                                 _p(b1), _p(Wu), _p(W2), _p(b2), _p(x), _p(Wsh_g), _p(Wsh_u),
                                 _p(Wsh_d), _p(y_perm), _p(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn")


def moe_combine(cfg, y_perm, row_of, y, ws, stream=None):
    _check(lib().moe_combine(ctypes.byref(cfg), _p(y_perm), _p(row_of), _p(y), _p(ws), ws.numel(),
                             _stream(stream)), "moe_combine")


def moe_balance_stats(cfg, counts, psum, f, P, loss, stream=None):
    _check(lib().moe_balance_stats(ctypes.byref(cfg), _p(counts), _p(psum), _p(f), _p(P), _p(loss),
                                   _stream(stream)), "moe_balance_stats")


def moe_forward(cfg, x, Wr, logit_bias, sel_bias, W1, b1, Wu, W2, b2, Wsh_g, Wsh_u, Wsh_d,
                y, idx, gate, counts, f, P, loss, logits_out, n_dropped, ws, stream=None):
    _check(lib().moe_forward(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias), _p(W1),
                             _p(b1), _p(Wu), _p(W2), _p(b2), _p(Wsh_g), _p(Wsh_u), _p(Wsh_d), _p(y),
                             _p(idx), _p(gate), _p(counts), _p(f), _p(P), _p(loss), _p(logits_out),
                             _p(n_dropped), _p(ws), ws.numel(), _stream(stream)), "moe_forward")


def moe_forward_train(cfg, x, Wr, logit_bias, sel_bias, W1, b1, Wu, W2, b2, Wsh_g, Wsh_u, Wsh_d,
                      y, idx, gate, counts, f, P, loss, logits_out, n_dropped, ws, bwd_ws, stream=None):
    _check(lib().moe_forward_train(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias), _p(W1),
                                   _p(b1), _p(Wu), _p(W2), _p(b2), _p(Wsh_g), _p(Wsh_u), _p(Wsh_d), _p(y),
                                   _p(idx), _p(gate), _p(counts), _p(f), _p(P), _p(loss), _p(logits_out),
                                   _p(n_dropped), _p(ws), ws.numel(), _p(bwd_ws), bwd_ws.numel(), _stream(stream)),
           "moe_forward_train")


def ep_workspace_size(cfg, n_src, max_rows) -> int:
    n = int(lib().moe_ep_workspace_size(ctypes.byref(cfg), int(n_src), int(max_rows)))
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_ep_workspace_size", last_error_detail())
    return n


def moe_ep_grouped_ffn(cfg, n_src, group_offsets, x_rows, row_gate, W1, b1, Wu, W2, b2, y_rows, ws, stream=None):
    """Grouped FFN over rows received from n_src sources: group src * E + e
    (rows group_offsets[g] .. group_offsets[g+1]) uses local expert e."""
    _check(lib().moe_ep_grouped_ffn(ctypes.byref(cfg), int(n_src), _p(group_offsets), int(x_rows.shape[0]),
                                    _p(x_rows), _p(row_gate), _p(W1), _p(b1), _p(Wu), _p(W2), _p(b2), _p(y_rows),
                                    _p(ws), ws.numel(), _stream(stream)), "moe_ep_grouped_ffn")


def backward_workspace_size(cfg) -> int:
    n = int(lib().moe_backward_workspace_size(ctypes.byref(cfg)))
    if n == 0:
        raise MoEError(MOE_ERR_UNSUPPORTED, "moe_backward_workspace_size", last_error_detail())
    return n


def moe_backward(cfg, x, Wr, W1, b1, Wu, W2, b2, Wsh_g, Wsh_u, Wsh_d, idx, gate, logits, counts, dy, alpha, dx, dWr,
                 dlogit_bias, dW1, db1, dWu, dW2, db2, dWsh_g, dWsh_u, dWsh_d, fwd_ws, ws, stream=None):
    _check(lib().moe_backward(ctypes.byref(cfg), _p(x), _p(Wr), _p(W1), _p(b1), _p(Wu), _p(W2), _p(b2), _p(Wsh_g),
                              _p(Wsh_u), _p(Wsh_d), _p(idx), _p(gate), _p(logits), _p(counts), _p(dy), float(alpha),
                              _p(dx), _p(dWr), _p(dlogit_bias), _p(dW1), _p(db1), _p(dWu), _p(dW2), _p(db2),
                              _p(dWsh_g), _p(dWsh_u), _p(dWsh_d), _p(fwd_ws), fwd_ws.numel(), _p(ws), ws.numel(),
                              _stream(stream)), "moe_backward")


def backward(cfg, inp, out, fwd_ws, dy, alpha=0.0, ws=None, stream=None) -> dict:
    """moe_backward after forward(cfg, inp, out, fwd_ws) (out must hold the
    router logits: Outputs(..., want_logits=True)).  Returns the gradients
    as fp32 tensors (dx in the layer dtype) keyed like the inputs."""
    if out.logits is None:
        raise ValueError("the backward pass needs the forward's router logits (Outputs(want_logits=True))")
    dev = dy.device
    T, d, E, F, S = cfg.T, cfg.d_model, cfg.E, cfg.d_ff, cfg.d_ff_shared
    f32 = dict(dtype=torch.float32, device=dev)
    swiglu = cfg.act == MOE_ACT_SWIGLU
    g = dict(dx=torch.empty((T, d), dtype=layer_dtype(cfg), device=dev), dWr=torch.empty((d, E), **f32),
             dlogit_bias=torch.empty(E, **f32), dW1=torch.empty((E, F, d), **f32),
             dWu=torch.empty((E, F, d), **f32) if swiglu else None, dW2=torch.empty((E, d, F), **f32),
             db1=None if swiglu else torch.empty((E, F), **f32), db2=None if swiglu else torch.empty((E, d), **f32),
             dWsg=torch.empty((S, d), **f32) if S else None, dWsu=torch.empty((S, d), **f32) if S and swiglu else None,
             dWsd=torch.empty((d, S), **f32) if S else None)
    if ws is None:
        ws = torch.empty(backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    moe_backward(cfg, inp["x"], inp["Wr"], inp["W1"], inp.get("b1"), inp.get("Wu"), inp["W2"], inp.get("b2"),
                 inp.get("Wsg"), inp.get("Wsu"), inp.get("Wsd"), out.idx, out.gate, out.logits, out.counts, dy, alpha,
                 g["dx"], g["dWr"], g["dlogit_bias"], g["dW1"], g["db1"], g["dWu"], g["dW2"], g["db2"], g["dWsg"],
                 g["dWsu"], g["dWsd"], fwd_ws, ws, stream)
    return g


def moe_workspace_view(cfg, ws) -> MoeWsView:
    v = MoeWsView()
    _check(lib().moe_workspace_view(ctypes.byref(cfg), _p(ws), ws.numel() * ws.element_size(), ctypes.byref(v)),
           "moe_workspace_view")
    return v


def workspace_tables(cfg, ws) -> dict:
    """The forward pass's dispatch tables and intermediate rows as tensors
    that alias the workspace (slices of `ws` at the addresses
    moe_workspace_view reports)."""
    v = moe_workspace_view(cfg, ws)
    base = ws.data_ptr()
    T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.top_k
    rows = perm_rows(cfg)
    dt = layer_dtype(cfg)

    def region(addr, n, dtype, shape):
        off = addr - base
        nbytes = n * torch.tensor([], dtype=dtype).element_size()
        return ws[off:off + nbytes].view(dtype).view(shape)

    return dict(kept=region(v.kept, E, torch.int32, (E,)),
                offsets=region(v.offsets, E + 1, torch.int32, (E + 1,)),
                row_of=region(v.row_of, T * k, torch.int32, (T, k)),
                row_token=region(v.row_token, T * k, torch.int32, (T * k,)),
                row_gate=region(v.row_gate, T * k, torch.float32, (T * k,)),
                x_perm=region(v.x_perm, T * k * d, dt, (T * k, d)),
                H=region(v.H, rows * v.h_stride, dt, (rows, v.h_stride)),
                y_perm=region(v.y_perm, rows * d, dt, (rows, d)))


def moe_bias_update(cfg, counts, sel_bias, gamma, stream=None):
    _check(lib().moe_bias_update(ctypes.byref(cfg), _p(counts), _p(sel_bias), float(gamma), _stream(stream)),
           "moe_bias_update")


def moe_routing_health(cfg, counts, P, out, stream=None):
    _check(lib().moe_routing_health(ctypes.byref(cfg), _p(counts), _p(P), _p(out), _stream(stream)),
           "moe_routing_health")


def moe_get_device_status(ws, stream=None) -> int:
    out = c_i32(0)
    _check(lib().moe_get_device_status(_p(ws), _stream(stream), ctypes.byref(out)),
           "moe_get_device_status")
    return int(out.value)


def moe_check_wait_timeout(ws, limit_ns, stream=None):
    """Launch the bounded-wait self-check (records MOE_ERR_TIMEOUT in ws)."""
    _check(lib().moe_check_wait_timeout(_p(ws), ctypes.c_uint64(int(limit_ns)), _stream(stream)),
           "moe_check_wait_timeout")


def layer_dtype(cfg):
    return torch.bfloat16 if cfg.dtype == MOE_BF16 else torch.float32


class Outputs:
    """Device output buffers of one moe_forward call (allocated once, reused)."""

    def __init__(self, cfg, device="cuda", want_logits=False):
        T, d, E, k = cfg.T, cfg.d_model, cfg.E, cfg.top_k
        self.y = torch.empty((T, d), dtype=layer_dtype(cfg), device=device)
        self.idx = torch.empty((T, k), dtype=torch.int32, device=device)
        self.gate = torch.empty((T, k), dtype=torch.float32, device=device)
        self.counts = torch.empty(E, dtype=torch.int32, device=device)
        self.f = torch.empty(E, dtype=torch.float32, device=device)
        self.P = torch.empty(E, dtype=torch.float32, device=device)
        self.loss = torch.empty(1, dtype=torch.float64, device=device)
        self.n_dropped = torch.zeros(1, dtype=torch.int32, device=device)
        self.logits = torch.empty((T, E), dtype=torch.float32, device=device) if want_logits else None


def forward(cfg, inp, out: Outputs, ws, stream=None):
    """moe_forward on a dict of device inputs (keys as in synthetic.generate)."""
    moe_forward(cfg, inp["x"], inp["Wr"], inp.get("logit_bias"), inp.get("sel_bias"),
                inp["W1"], inp.get("b1"), inp.get("Wu"), inp["W2"], inp.get("b2"),
                inp.get("Wsg"), inp.get("Wsu"), inp.get("Wsd"),
                out.y, out.idx, out.gate, out.counts, out.f, out.P, out.loss, out.logits,
                out.n_dropped, ws, stream)


def alloc_backward_workspace(cfg, device="cuda") -> torch.Tensor:
    return torch.empty(backward_workspace_size(cfg), dtype=torch.uint8, device=device)


def forward_train(cfg, inp, out: Outputs, ws, bwd_ws, stream=None):
    """moe_forward_train: forward(...) that also leaves the expert
    pre-activations in bwd_ws for the following backward(..., ws=bwd_ws)."""
    moe_forward_train(cfg, inp["x"], inp["Wr"], inp.get("logit_bias"), inp.get("sel_bias"),
                      inp["W1"], inp.get("b1"), inp.get("Wu"), inp["W2"], inp.get("b2"),
                      inp.get("Wsg"), inp.get("Wsu"), inp.get("Wsd"),
                      out.y, out.idx, out.gate, out.counts, out.f, out.P, out.loss, out.logits,
                      out.n_dropped, ws, bwd_ws, stream)


# ---------------------------------------------------------------- FP8 experts
FP8_WEIGHTS = ("W1", "Wu", "W2", "Wsg", "Wsu", "Wsd")
_FP8_FIELD = {"W1": "W1", "Wu": "Wu", "W2": "W2", "Wsg": "Wsh_g", "Wsu": "Wsh_u", "Wsd": "Wsh_d"}


def fp8_experts(w) -> MoeFp8Experts:
    """moe_fp8_experts from a dict of device tensors: e4m3 codes (uint8)
    under W1, Wu, W2, Wsg, Wsu, Wsd and fp32 scales under "<name>_scale"."""
    s = MoeFp8Experts()
    for name in FP8_WEIGHTS:
        field = _FP8_FIELD[name]
        setattr(s, field, _p(w.get(name)))
        setattr(s, field + "_scale", _p(w.get(name + "_scale")))
    return s


def moe_quantize_rows_e4m3(x, codes, scale, rows=None, cols=None, ld_in=None, ld_out=None, stream=None):
    """Per-row e4m3 quantization of a bf16 [rows, cols] tensor into codes
    (uint8, same shape unless ld_out is given) and scale [rows] fp32."""
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld_in = x.shape[1] if ld_in is None else ld_in
    ld_out = codes.shape[1] if ld_out is None else ld_out
    _check(lib().moe_quantize_rows_e4m3(_p(x), rows, cols, ld_in, _p(codes), ld_out, _p(scale), _stream(stream)),
           "moe_quantize_rows_e4m3")


def moe_grouped_ffn_fp8(cfg, x8_perm, x8_perm_scale, offsets, row_gate, w, b1, b2, x8, x8_scale, y_perm, ws,
                        stream=None):
    ex = fp8_experts(w)
    _check(lib().moe_grouped_ffn_fp8(ctypes.byref(cfg), _p(x8_perm), _p(x8_perm_scale), _p(offsets), _p(row_gate),
                                     ctypes.byref(ex), _p(b1), _p(b2), _p(x8), _p(x8_scale), _p(y_perm), _p(ws),
                                     ws.numel(), _stream(stream)), "moe_grouped_ffn_fp8")


def moe_forward_fp8(cfg, x, Wr, logit_bias, sel_bias, w, b1, b2, y, idx, gate, counts, f, P, loss, logits_out,
                    n_dropped, ws, stream=None):
    ex = fp8_experts(w)
    _check(lib().moe_forward_fp8(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias), ctypes.byref(ex),
                                 _p(b1), _p(b2), _p(y), _p(idx), _p(gate), _p(counts), _p(f), _p(P), _p(loss),
                                 _p(logits_out), _p(n_dropped), _p(ws), ws.numel(), _stream(stream)),
           "moe_forward_fp8")


def moe_router_freeze(cfg, Wr, ws, stream=None):
    """Split W_r into the workspace once; later router calls on ws with the
    same W_r pointer skip the split (see include/moe.h)."""
    _check(lib().moe_router_freeze(ctypes.byref(cfg), _p(Wr), _p(ws), ws.numel(), _stream(stream)),
           "moe_router_freeze")


# ---------------------------------------------------------------- MX experts
def mx_sld(cfg) -> int:
    """Smallest valid scale row stride (bytes) for a configuration."""
    need = max(cfg.d_model, cfg.d_ff, cfg.d_ff_shared) // 32
    return (need + 15) // 16 * 16


def mx_experts(w, sld) -> MoeMxExperts:
    """moe_mx_experts from a dict of device tensors: e4m3 codes (uint8) under
    W1, Wu, W2, Wsg, Wsu, Wsd and scale bytes (uint8, rows of sld bytes) under
    "<name>_scale"."""
    s = MoeMxExperts()
    for name in FP8_WEIGHTS:
        field = _FP8_FIELD[name]
        setattr(s, field, _p(w.get(name)))
        setattr(s, field + "_scale", _p(w.get(name + "_scale")))
    s.sld = int(sld)
    return s


def moe_quantize_rows_mx(x, codes, scales, rows=None, cols=None, ld_in=None, ld_out=None, ld_scale=None,
                         stream=None):
    """MX quantization of a bf16 [rows, cols] tensor into codes (uint8) and
    scale bytes (uint8 [rows, ld_scale])."""
    rows = x.shape[0] if rows is None else rows
    cols = x.shape[1] if cols is None else cols
    ld_in = x.shape[1] if ld_in is None else ld_in
    ld_out = codes.shape[1] if ld_out is None else ld_out
    ld_scale = scales.shape[1] if ld_scale is None else ld_scale
    _check(lib().moe_quantize_rows_mx(_p(x), rows, cols, ld_in, _p(codes), ld_out, _p(scales), ld_scale,
                                      _stream(stream)), "moe_quantize_rows_mx")


def grouped_ffn_mx_workspace_size(cfg, sld) -> int:
    return int(lib().moe_grouped_ffn_mx_workspace_size(ctypes.byref(cfg), int(sld)))


def moe_grouped_ffn_mx(cfg, x8_perm, xs_perm, offsets, row_gate, w, sld, b1, b2, x8, xs, y_perm, ws, stream=None):
    ex = mx_experts(w, sld)
    _check(lib().moe_grouped_ffn_mx(ctypes.byref(cfg), _p(x8_perm), _p(xs_perm), _p(offsets), _p(row_gate),
                                    ctypes.byref(ex), _p(b1), _p(b2), _p(x8), _p(xs), _p(y_perm), _p(ws),
                                    ws.numel(), _stream(stream)), "moe_grouped_ffn_mx")


def moe_forward_mx(cfg, x, Wr, logit_bias, sel_bias, w, sld, b1, b2, y, idx, gate, counts, f, P, loss, logits_out,
                   n_dropped, ws, mx_ws, stream=None):
    ex = mx_experts(w, sld)
    _check(lib().moe_forward_mx(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias), ctypes.byref(ex),
                                _p(b1), _p(b2), _p(y), _p(idx), _p(gate), _p(counts), _p(f), _p(P), _p(loss),
                                _p(logits_out), _p(n_dropped), _p(ws), ws.numel(), _p(mx_ws), mx_ws.numel(),
                                _stream(stream)), "moe_forward_mx")


def alloc_mx_workspace(cfg, sld, device="cuda") -> torch.Tensor:
    """A zeroed MX workspace (moe_grouped_ffn_mx_workspace_size bytes)."""
    n = grouped_ffn_mx_workspace_size(cfg, sld)
    if n == 0:
        raise MoEError(MOE_ERR_INVALID_ARG, "moe_grouped_ffn_mx_workspace_size", last_error_detail())
    return torch.zeros(n, dtype=torch.uint8, device=device)


def forward_mx(cfg, inp, wmx, sld, out: Outputs, ws, mx_ws, stream=None):
    """moe_forward_mx on a dict of device inputs and a dict of MX experts."""
    moe_forward_mx(cfg, inp["x"], inp["Wr"], inp.get("logit_bias"), inp.get("sel_bias"), wmx, sld,
                   wmx.get("b1"), wmx.get("b2"), out.y, out.idx, out.gate, out.counts, out.f, out.P, out.loss,
                   out.logits, out.n_dropped, ws, mx_ws, stream)


# ---------------------------------------------------------------- INT4 weight-only experts
def w4_sld(cfg) -> int:
    """Smallest valid bf16 scale row stride (bytes) for a configuration."""
    need = max(cfg.d_model, cfg.d_ff, cfg.d_ff_shared) // 64
    return (need + 15) // 16 * 16


def w4_experts(w, sld) -> MoeW4Experts:
    """moe_w4_experts from a dict of device tensors: packed codes (uint8) under
    W1, Wu, W2, Wsg, Wsu, Wsd and bf16 scales as bytes (uint8, rows of sld
    bytes) under "<name>_scale"."""
    s = MoeW4Experts()
    for name in FP8_WEIGHTS:
        field = _FP8_FIELD[name]
        setattr(s, field, _p(w.get(name)))
        setattr(s, field + "_scale", _p(w.get(name + "_scale")))
    s.sld = int(sld)
    return s


def moe_grouped_ffn_w4(cfg, x_perm, offsets, row_gate, w, sld, b1, b2, x, y_perm, ws, stream=None):
    ex = w4_experts(w, sld)
    _check(lib().moe_grouped_ffn_w4(ctypes.byref(cfg), _p(x_perm), _p(offsets), _p(row_gate), ctypes.byref(ex),
                                    _p(b1), _p(b2), _p(x), _p(y_perm), _p(ws), ws.numel(), _stream(stream)),
           "moe_grouped_ffn_w4")


def moe_forward_w4(cfg, x, Wr, logit_bias, sel_bias, w, sld, b1, b2, y, idx, gate, counts, f, P, loss, logits_out,
                   n_dropped, ws, stream=None):
    ex = w4_experts(w, sld)
    _check(lib().moe_forward_w4(ctypes.byref(cfg), _p(x), _p(Wr), _p(logit_bias), _p(sel_bias), ctypes.byref(ex),
                                _p(b1), _p(b2), _p(y), _p(idx), _p(gate), _p(counts), _p(f), _p(P), _p(loss),
                                _p(logits_out), _p(n_dropped), _p(ws), ws.numel(), _stream(stream)),
           "moe_forward_w4")


def forward_w4(cfg, inp, w4, sld, out: Outputs, ws, stream=None):
    """moe_forward_w4 on a dict of device inputs and a dict of INT4 experts."""
    moe_forward_w4(cfg, inp["x"], inp["Wr"], inp.get("logit_bias"), inp.get("sel_bias"), w4, sld,
                   w4.get("b1"), w4.get("b2"), out.y, out.idx, out.gate, out.counts, out.f, out.P, out.loss,
                   out.logits, out.n_dropped, ws, stream)


def forward_fp8(cfg, inp, w8, out: Outputs, ws, stream=None):
    """moe_forward_fp8 on a dict of device inputs and a dict of FP8 experts."""
    moe_forward_fp8(cfg, inp["x"], inp["Wr"], inp.get("logit_bias"), inp.get("sel_bias"), w8,
                    inp.get("b1"), inp.get("b2"), out.y, out.idx, out.gate, out.counts, out.f, out.P, out.loss,
                    out.logits, out.n_dropped, ws, stream)
