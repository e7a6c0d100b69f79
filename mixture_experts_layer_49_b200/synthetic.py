"""Seeded synthetic workloads for the MoE layer forward pass.

This module only draws random numbers with the shapes and distributions of
the layers the pages describe; it contains none of the layer's arithmetic.
Both the CUDA path (benchmark, tests) and the CPU oracle (tests) are fed from
it.

Distributions:
  x      ~ N(0, 1), stored in the layer dtype (bf16 or fp32)
  W_r    ~ N(0, 1/d_model), fp32, layout [d_model, E]
  W_in   ~ N(0, 1/d_model)  (GELU W1, SwiGLU W_gate and W_up)  [E, d_ff, d_model]
  W_out  ~ N(0, 1/d_ff)     (GELU W2, SwiGLU W_down)           [E, d_model, d_ff]
  b1, b2 ~ U(-0.01, 0.01), fp32 (GELU experts only)
  logit skew (an additive per-expert router offset):
    "normal": beta_e ~ N(0, 1)
    "zipf":   beta_e = log(r_e^-1.1 / sum_r r^-1.1), r a seeded permutation of 1..E
  selection bias b_e ~ N(0, sel_bias_std)   (auxiliary-loss-free routing)

Every tensor has its own generator stream, keyed by (seed, workload name,
tensor name, part), so one tensor (or one expert's slice) can be regenerated
alone.  Large weight tensors are drawn one expert at a time.
"""
from __future__ import annotations

import dataclasses
import zlib

import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    d_model: int
    E: int
    d_ff: int
    top_k: int
    dtype: str = "bf16"              # "bf16" or "f32"
    act: str = "swiglu"              # "swiglu" or "gelu" (GELU experts carry biases)
    score: str = "softmax"           # "softmax" or "sigmoid"
    renorm: int = 1                  # softmax: renormalise gates over the top-k
    capacity_factor: float = 0.0     # <= 0: no capacity limit
    d_ff_shared: int = 0             # 0: no shared expert
    logit_skew: str = "none"         # "none", "normal", "zipf"
    sel_bias_std: float = 0.0        # > 0: draw an aux-loss-free selection bias

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)

    def routed_rows(self) -> int:
        return self.T * self.top_k

    def expert_flops(self, kept_rows: int) -> float:
        """Multiply-add FLOPs of the expert FFNs over `kept_rows` routed rows
        plus the shared expert over all tokens."""
        mats = 3 if self.act == "swiglu" else 2
        f = 2.0 * kept_rows * self.d_model * self.d_ff * mats
        if self.d_ff_shared:
            f += 2.0 * self.T * self.d_model * self.d_ff_shared * mats
        return f


WORKLOADS = {
    # Tiny fp32 layer: Linear(128->256)+GELU+Linear(256->128) experts with bias.
    "tiny_fp32": Workload("tiny_fp32", T=256, d_model=128, E=8, d_ff=256, top_k=2,
                          dtype="f32", act="gelu", score="softmax", renorm=1),
    # Switch-style top-1 with capacity factor 1.25 and skewed router.
    "switch_top1": Workload("switch_top1", T=8192, d_model=1024, E=16, d_ff=4096, top_k=1,
                            act="gelu", renorm=0, capacity_factor=1.25, logit_skew="normal"),
    # Mixtral-shaped layer.
    "mixtral": Workload("mixtral", T=4096, d_model=4096, E=8, d_ff=14336, top_k=2),
    # Qwen3-MoE-shaped layer with Zipf(1.1) expert popularity.
    "qwen3_moe": Workload("qwen3_moe", T=16384, d_model=2048, E=128, d_ff=768, top_k=8,
                          logit_skew="zipf"),
    # DeepSeek-V3-shaped layer: sigmoid scores, selection bias, shared expert.
    "deepseek_v3": Workload("deepseek_v3", T=8192, d_model=7168, E=256, d_ff=2048, top_k=8,
                            score="sigmoid", d_ff_shared=2048, sel_bias_std=0.1),
}


def stream_seed(seed: int, workload: str, tensor: str, part: int = 0) -> int:
    key = ("%d/%s/%s/%d" % (seed, workload, tensor, part)).encode()
    return (zlib.crc32(key) << 20) ^ (zlib.crc32(key[::-1]) & 0xFFFFF) ^ (seed * 0x9E3779B1)


def _gen(device, seed, wl, tensor, part=0):
    g = torch.Generator(device=device)
    g.manual_seed(stream_seed(seed, wl.name, tensor, part) & ((1 << 62) - 1))
    return g


def _normal(shape, std, dtype, device, g):
    t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        t.mul_(std)
    return t.to(dtype)


def _tdtype(wl):
    return torch.float32 if wl.dtype == "f32" else torch.bfloat16


def _stacked(wl, name, E, rows, cols, std, device, seed):
    out = torch.empty((E, rows, cols), dtype=_tdtype(wl), device=device)
    for e in range(E):
        out[e].copy_(_normal((rows, cols), std, _tdtype(wl), device, _gen(device, seed, wl, name, e)))
    return out


def generate(wl: Workload, device="cpu", seed: int = 0, weights: bool = True) -> dict:
    """Draw all inputs of one layer call.  Keys:
    x, Wr, logit_bias, sel_bias, W1 (GELU W1 / SwiGLU W_gate), Wu (SwiGLU W_up),
    W2 (W2 / W_down), b1, b2, Wsg, Wsu, Wsd (shared expert).  Absent ones are None."""
    dev = torch.device(device)
    dt = _tdtype(wl)
    d, E, F = wl.d_model, wl.E, wl.d_ff
    inp = dict(workload=wl)
    inp["x"] = _normal((wl.T, d), 1.0, dt, dev, _gen(dev, seed, wl, "x"))
    inp["Wr"] = _normal((d, E), d ** -0.5, torch.float32, dev, _gen(dev, seed, wl, "Wr"))
    if wl.logit_skew == "normal":
        inp["logit_bias"] = _normal((E,), 1.0, torch.float32, dev, _gen(dev, seed, wl, "skew"))
    elif wl.logit_skew == "zipf":
        g = _gen(torch.device("cpu"), seed, wl, "skew")
        ranks = (torch.randperm(E, generator=g) + 1).to(torch.float64)
        w = ranks.pow(-1.1)
        inp["logit_bias"] = torch.log(w / w.sum()).to(torch.float32).to(dev)
    else:
        inp["logit_bias"] = None
    inp["sel_bias"] = (_normal((E,), wl.sel_bias_std, torch.float32, dev, _gen(dev, seed, wl, "selb"))
                       if wl.sel_bias_std > 0 else None)
    for key in ("W1", "Wu", "W2", "b1", "b2", "Wsg", "Wsu", "Wsd"):
        inp[key] = None
    if not weights:
        return inp
    inp["W1"] = _stacked(wl, "W1", E, F, d, d ** -0.5, dev, seed)
    inp["W2"] = _stacked(wl, "W2", E, d, F, F ** -0.5, dev, seed)
    if wl.act == "swiglu":
        inp["Wu"] = _stacked(wl, "Wu", E, F, d, d ** -0.5, dev, seed)
    else:
        g = _gen(dev, seed, wl, "b1")
        inp["b1"] = (torch.rand((E, F), generator=g, device=dev) * 0.02 - 0.01)
        g = _gen(dev, seed, wl, "b2")
        inp["b2"] = (torch.rand((E, d), generator=g, device=dev) * 0.02 - 0.01)
    if wl.d_ff_shared:
        S = wl.d_ff_shared
        inp["Wsg"] = _normal((S, d), d ** -0.5, dt, dev, _gen(dev, seed, wl, "Wsg"))
        inp["Wsd"] = _normal((d, S), S ** -0.5, dt, dev, _gen(dev, seed, wl, "Wsd"))
        if wl.act == "swiglu":
            inp["Wsu"] = _normal((S, d), d ** -0.5, dt, dev, _gen(dev, seed, wl, "Wsu"))
    return inp


def redraw_rows(x: torch.Tensor, rows, wl: Workload, seed: int, attempt: int) -> None:
    """Replace rows of x (in place) with fresh N(0,1) draws from a sub-stream
    keyed by the attempt number (used to enforce a selection margin)."""
    rows = torch.as_tensor(rows, dtype=torch.long)
    if rows.numel() == 0:
        return
    g = _gen(x.device, seed, wl, "x-redraw", attempt)
    fresh = torch.randn((rows.numel(), x.shape[1]), generator=g, device=x.device, dtype=torch.float32)
    x[rows.to(x.device)] = fresh.to(x.dtype)


def to_numpy_raw(t: torch.Tensor):
    """Host numpy view of a tensor: bf16 becomes its uint16 bit patterns."""
    if t is None:
        return None
    t = t.detach().to("cpu").contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view("uint16")
    return t.numpy()


def _fp8_stack(wl, name, E, rows, cols, device, seed):
    """E x rows x cols e4m3 codes of N(0, 1) draws (through torch's
    float8_e4m3fn cast) and E x rows scales U(0.5, 1.5) / sqrt(cols)."""
    codes = torch.empty((E, rows, cols), dtype=torch.uint8, device=device)
    scale = torch.empty((E, rows), dtype=torch.float32, device=device)
    for e in range(E):
        g = _gen(device, seed, wl, name + "_e4m3", e)
        codes[e].copy_(torch.randn((rows, cols), generator=g, device=device).to(torch.float8_e4m3fn)
                       .view(torch.uint8))
        scale[e].copy_((torch.rand((rows,), generator=g, device=device) + 0.5) * cols ** -0.5)
    return codes, scale


def _mx_stack(wl, name, E, rows, cols, sld, device, seed):
    """E x rows x cols e4m3 codes of N(0, 1) draws (torch's float8_e4m3fn
    cast) and E x rows x sld scale bytes: one per 32 inputs, uniform over the
    three powers of two around 1/sqrt(cols), bytes past cols / 32 zero."""
    codes = torch.empty((E, rows, cols), dtype=torch.uint8, device=device)
    scale = torch.zeros((E, rows, sld), dtype=torch.uint8, device=device)
    base = 127 - int(math.ceil(math.log2(math.sqrt(cols))))
    for e in range(E):
        g = _gen(device, seed, wl, name + "_mx", e)
        codes[e].copy_(torch.randn((rows, cols), generator=g, device=device).to(torch.float8_e4m3fn)
                       .view(torch.uint8))
        scale[e, :, :cols // 32].copy_(torch.randint(base - 1, base + 2, (rows, cols // 32), generator=g,
                                                     device=device).to(torch.uint8))
    return codes, scale


def generate_mx_experts(wl: Workload, sld: int, device="cpu", seed: int = 0) -> dict:
    """Block-scaled (MX) expert weights for a bf16 workload: e4m3 codes
    (uint8, nn.Linear [out, in] layout) and E8M0 scale bytes, one per 32
    inputs, in rows of sld bytes.  Keys W1, Wu, W2, Wsg, Wsu, Wsd and
    "<key>_scale" (absent ones None), and for GELU experts the fp32 biases b1,
    b2 (the same draws as generate()'s)."""
    dev = torch.device(device)
    d, E, F = wl.d_model, wl.E, wl.d_ff
    w = {k: None for k in ("W1", "Wu", "W2", "Wsg", "Wsu", "Wsd")}
    w.update({k + "_scale": None for k in list(w)})
    w["W1"], w["W1_scale"] = _mx_stack(wl, "W1", E, F, d, sld, dev, seed)
    w["W2"], w["W2_scale"] = _mx_stack(wl, "W2", E, d, F, sld, dev, seed)
    if wl.act == "swiglu":
        w["Wu"], w["Wu_scale"] = _mx_stack(wl, "Wu", E, F, d, sld, dev, seed)
    if wl.act == "gelu":
        g = _gen(dev, seed, wl, "b1")
        w["b1"] = (torch.rand((E, F), generator=g, device=dev) * 0.02 - 0.01)
        g = _gen(dev, seed, wl, "b2")
        w["b2"] = (torch.rand((E, d), generator=g, device=dev) * 0.02 - 0.01)
    if wl.d_ff_shared:
        S = wl.d_ff_shared
        c, s = _mx_stack(wl, "Wsg", 1, S, d, sld, dev, seed)
        w["Wsg"], w["Wsg_scale"] = c[0], s[0]
        c, s = _mx_stack(wl, "Wsd", 1, d, S, sld, dev, seed)
        w["Wsd"], w["Wsd_scale"] = c[0], s[0]
        if wl.act == "swiglu":
            c, s = _mx_stack(wl, "Wsu", 1, S, d, sld, dev, seed)
            w["Wsu"], w["Wsu_scale"] = c[0], s[0]
    return w


def _w4_stack(wl, name, E, rows, cols, sld, device, seed):
    """E x rows x cols/2 packed INT4 codes (uniform bytes: every nibble uniform
    over -8..7) and E x rows x sld scale bytes: one bf16 scale per 128 inputs,
    U(0.5, 1.5) / (3 sqrt(cols)) (so the weights spread like N(0, 1/cols)),
    bytes past the scales zero."""
    codes = torch.empty((E, rows, cols // 2), dtype=torch.uint8, device=device)
    scale = torch.zeros((E, rows, sld), dtype=torch.uint8, device=device)
    ng = cols // 128
    for e in range(E):
        g = _gen(device, seed, wl, name + "_w4", e)
        codes[e].copy_(torch.randint(0, 256, (rows, cols // 2), generator=g, device=device).to(torch.uint8))
        s = (torch.rand((rows, ng), generator=g, device=device) + 0.5) / (3.0 * math.sqrt(cols))
        scale[e, :, :2 * ng].copy_(s.to(torch.bfloat16).view(torch.uint8).reshape(rows, 2 * ng))
    return codes, scale


def generate_w4_experts(wl: Workload, sld: int, device="cpu", seed: int = 0) -> dict:
    """INT4 weight-only expert weights for a bf16 workload: packed codes
    (uint8, nn.Linear [out, in/2] layout, low nibble = even input) and bf16
    group scales as bytes, one per 128 inputs, in rows of sld bytes.  Keys
    W1, Wu, W2, Wsg, Wsu, Wsd and "<key>_scale" (absent ones None), and for
    GELU experts the fp32 biases b1, b2 (the same draws as generate()'s)."""
    dev = torch.device(device)
    d, E, F = wl.d_model, wl.E, wl.d_ff
    w = {k: None for k in ("W1", "Wu", "W2", "Wsg", "Wsu", "Wsd")}
    w.update({k + "_scale": None for k in list(w)})
    w["W1"], w["W1_scale"] = _w4_stack(wl, "W1", E, F, d, sld, dev, seed)
    w["W2"], w["W2_scale"] = _w4_stack(wl, "W2", E, d, F, sld, dev, seed)
    if wl.act == "swiglu":
        w["Wu"], w["Wu_scale"] = _w4_stack(wl, "Wu", E, F, d, sld, dev, seed)
    if wl.act == "gelu":
        g = _gen(dev, seed, wl, "b1")
        w["b1"] = (torch.rand((E, F), generator=g, device=dev) * 0.02 - 0.01)
        g = _gen(dev, seed, wl, "b2")
        w["b2"] = (torch.rand((E, d), generator=g, device=dev) * 0.02 - 0.01)
    if wl.d_ff_shared:
        S = wl.d_ff_shared
        c, s = _w4_stack(wl, "Wsg", 1, S, d, sld, dev, seed)
        w["Wsg"], w["Wsg_scale"] = c[0], s[0]
        c, s = _w4_stack(wl, "Wsd", 1, d, S, sld, dev, seed)
        w["Wsd"], w["Wsd_scale"] = c[0], s[0]
        if wl.act == "swiglu":
            c, s = _w4_stack(wl, "Wsu", 1, S, d, sld, dev, seed)
            w["Wsu"], w["Wsu_scale"] = c[0], s[0]
    return w


def generate_fp8_experts(wl: Workload, device="cpu", seed: int = 0) -> dict:
    """FP8 expert weights for a bf16 workload: e4m3 codes (uint8, nn.Linear
    [out, in] layout) with one fp32 scale per output channel, spread like the
    bf16 weights (N(0, 1/fan_in)).  Keys W1, Wu, W2, Wsg, Wsu, Wsd and
    "<key>_scale" (absent ones None), and for GELU experts the fp32 biases
    b1, b2 (the same draws as generate()'s)."""
    dev = torch.device(device)
    d, E, F = wl.d_model, wl.E, wl.d_ff
    w = {k: None for k in ("W1", "Wu", "W2", "Wsg", "Wsu", "Wsd")}
    w.update({k + "_scale": None for k in list(w)})
    w["W1"], w["W1_scale"] = _fp8_stack(wl, "W1", E, F, d, dev, seed)
    w["W2"], w["W2_scale"] = _fp8_stack(wl, "W2", E, d, F, dev, seed)
    if wl.act == "swiglu":
        w["Wu"], w["Wu_scale"] = _fp8_stack(wl, "Wu", E, F, d, dev, seed)
    if wl.act == "gelu":            # the GELU experts' fp32 biases, as generate() draws them
        g = _gen(dev, seed, wl, "b1")
        w["b1"] = (torch.rand((E, F), generator=g, device=dev) * 0.02 - 0.01)
        g = _gen(dev, seed, wl, "b2")
        w["b2"] = (torch.rand((E, d), generator=g, device=dev) * 0.02 - 0.01)
    if wl.d_ff_shared:
        S = wl.d_ff_shared
        c, s = _fp8_stack(wl, "Wsg", 1, S, d, dev, seed)
        w["Wsg"], w["Wsg_scale"] = c[0], s[0]
        c, s = _fp8_stack(wl, "Wsd", 1, d, S, dev, seed)
        w["Wsd"], w["Wsd_scale"] = c[0], s[0]
        if wl.act == "swiglu":
            c, s = _fp8_stack(wl, "Wsu", 1, S, d, dev, seed)
            w["Wsu"], w["Wsu_scale"] = c[0], s[0]
    return w
