"""The C ABI without a GPU: the library loads, exports every symbol that
include/moe.h declares, and its host-side checks reject bad arguments before
any CUDA call (none of these calls reaches a launch)."""
import ctypes
import os
import re

import pytest
import torch

from mixture_experts_layer_49_b200 import native as nat

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe.h")


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"MOE_API\s+[\w\s\*]+?\b(moe_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    syms = declared_symbols()
    for name in ("moe_router_topk", "moe_permute", "moe_grouped_ffn", "moe_combine",
                 "moe_forward", "moe_balance_stats"):
        assert name in syms
    assert set(syms) == set(nat.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = nat.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name
    # nothing else is exported from the library's C namespace
    out = os.popen("nm -D --defined-only %s" % nat._build.LIB).read()
    exported = set(re.findall(r" T (moe_\w+)", out))
    assert exported == set(declared_symbols())


def cfg(**kw):
    base = dict(T=64, d_model=128, E=8, d_ff=256, top_k=2)
    base.update({k: kw.pop(k) for k in list(kw) if k in base})
    return nat.make_config(base["T"], base["d_model"], base["E"], base["d_ff"], base["top_k"], **kw)


def test_sizes_and_capacity():
    c = cfg()
    assert nat.workspace_size(c) > 0
    assert nat.router_blocks(c) == 2                     # 32 tokens per router block
    assert nat.router_blocks(cfg(T=300)) == 10
    assert nat.router_blocks(cfg(dtype="f32")) == 2
    assert nat.perm_rows(c) == 128
    assert nat.perm_rows(cfg(d_ff_shared=64)) == 128 + 64
    assert nat.capacity(c) == -1
    assert nat.capacity(cfg(T=8192, d_model=1024, E=16, d_ff=4096, top_k=1, capacity_factor=1.25)) == 640
    assert nat.capacity(cfg(T=7, E=3, top_k=2, capacity_factor=1.25)) == 5
    big = nat.workspace_size(cfg(T=1024))
    assert big > nat.workspace_size(c)


@pytest.mark.parametrize("kw,code", [
    (dict(T=-1), nat.MOE_ERR_INVALID_ARG),
    (dict(E=0), nat.MOE_ERR_INVALID_ARG),
    (dict(E=300), nat.MOE_ERR_UNSUPPORTED),
    (dict(top_k=0), nat.MOE_ERR_INVALID_ARG),
    (dict(top_k=9), nat.MOE_ERR_INVALID_ARG),
    (dict(E=64, top_k=33), nat.MOE_ERR_UNSUPPORTED),
    (dict(d_model=100), nat.MOE_ERR_UNSUPPORTED),
    (dict(d_ff=0), nat.MOE_ERR_INVALID_ARG),
    (dict(d_ff_shared=12), nat.MOE_ERR_UNSUPPORTED),
    (dict(renorm=2), nat.MOE_ERR_INVALID_ARG),
])
def test_bad_config_is_rejected(kw, code):
    c = cfg(**kw)
    assert nat.workspace_size(c) == 0
    rc = nat.lib().moe_balance_stats(ctypes.byref(c), *([ctypes.c_void_p(256)] * 5), None)
    assert rc == code, nat.last_error_detail()


def fake(n=1):
    return ctypes.c_void_p(4096 * n)


def forward_raw(c, ws=None, ws_bytes=None, **null):
    args = dict(x=fake(), Wr=fake(), lb=None, sb=None, W1=fake(), b1=None, Wu=fake(), W2=fake(), b2=None,
                Wsg=None, Wsu=None, Wsd=None, y=fake(), idx=fake(), gate=fake(), counts=fake(), f=fake(),
                P=fake(), loss=fake(), logits=None, nd=None)
    for k in null:
        args[k] = None
    if ws is None:
        ws = fake(16)
    if ws_bytes is None:
        ws_bytes = nat.workspace_size(c)
    return nat.lib().moe_forward(ctypes.byref(c), *args.values(), ws, ws_bytes, None)


@pytest.mark.parametrize("missing", ["x", "Wr", "W1", "Wu", "W2", "y", "idx", "gate", "counts", "loss"])
def test_null_pointer_is_rejected(missing):
    assert forward_raw(cfg(), **{missing: None}) == nat.MOE_ERR_INVALID_ARG
    assert missing.lower() in nat.last_error_detail().lower() or missing in nat.last_error_detail()


def test_shared_expert_weights_are_required():
    c = cfg(d_ff_shared=64)
    assert forward_raw(c) == nat.MOE_ERR_INVALID_ARG


def test_workspace_checks():
    c = cfg()
    assert forward_raw(c, ws_bytes=nat.workspace_size(c) - 1) == nat.MOE_ERR_WORKSPACE
    assert forward_raw(c, ws=ctypes.c_void_p(4096 + 16)) == nat.MOE_ERR_WORKSPACE
    assert nat.lib().moe_workspace_init(None, 1024, None) == nat.MOE_ERR_WORKSPACE
    out = ctypes.c_int32(0)
    assert nat.lib().moe_get_device_status(None, None, ctypes.byref(out)) == nat.MOE_ERR_WORKSPACE


def test_wait_timeout_check_arguments():
    L = nat.lib()
    assert L.moe_check_wait_timeout(None, 1000000, None) == nat.MOE_ERR_WORKSPACE
    assert L.moe_check_wait_timeout(ctypes.c_void_p(4096 + 16), 1000000, None) == nat.MOE_ERR_WORKSPACE
    assert L.moe_check_wait_timeout(ctypes.c_void_p(4096), 10, None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_check_wait_timeout(ctypes.c_void_p(4096), 20 * 10**9, None) == nat.MOE_ERR_INVALID_ARG


def test_status_strings():
    for s in range(7):
        assert nat.status_string(s) != "unknown status"
    assert nat.status_string(99) == "unknown status"


def test_binding_refuses_host_tensors():
    c = cfg()
    with pytest.raises(ValueError):
        nat.moe_combine(c, torch.zeros(4), torch.zeros(4, dtype=torch.int32), torch.zeros(4),
                        torch.zeros(256, dtype=torch.uint8))


def fp8_raw(c, w=None, **null):
    if w is None:
        w = nat.MoeFp8Experts(W1=4096, W1_scale=4096, Wu=4096, Wu_scale=4096, W2=4096, W2_scale=4096)
    args = dict(x=fake(), Wr=fake(), lb=None, sb=None)
    rest = dict(b1=None, b2=None, y=fake(), idx=fake(), gate=fake(), counts=fake(), f=fake(), P=fake(),
                loss=fake(), logits=None, nd=None)
    for k in null:
        (args if k in args else rest)[k] = None
    return nat.lib().moe_forward_fp8(ctypes.byref(c), *args.values(), ctypes.byref(w), *rest.values(), fake(16),
                                     nat.workspace_size(c), None)


def test_fp8_entry_points_check_arguments():
    # FP8 experts need a bf16 layer and widths that are multiples of 16
    assert fp8_raw(cfg(dtype="f32")) == nat.MOE_ERR_UNSUPPORTED
    assert fp8_raw(cfg(d_model=136)) == nat.MOE_ERR_UNSUPPORTED
    assert fp8_raw(cfg(d_ff=264)) == nat.MOE_ERR_UNSUPPORTED
    assert fp8_raw(cfg(d_ff_shared=24)) == nat.MOE_ERR_UNSUPPORTED
    # missing weights, scales or outputs
    assert fp8_raw(cfg(), w=nat.MoeFp8Experts(W1=4096, W2=4096, W2_scale=4096, Wu=4096, Wu_scale=4096)) \
        == nat.MOE_ERR_INVALID_ARG
    assert "W1_scale" in nat.last_error_detail()
    assert fp8_raw(cfg(), w=nat.MoeFp8Experts(W1=4096, W1_scale=4096, W2=4096, W2_scale=4096)) \
        == nat.MOE_ERR_INVALID_ARG                        # SwiGLU without W_up
    assert fp8_raw(cfg(d_ff_shared=64)) == nat.MOE_ERR_INVALID_ARG      # no shared expert weights
    assert fp8_raw(cfg(), y=None) == nat.MOE_ERR_INVALID_ARG
    # the weights struct is required even for an empty batch
    c0 = cfg(T=0)
    assert nat.lib().moe_forward_fp8(ctypes.byref(c0), None, None, None, None, None, None, None, None, None,
                                     None, fake(), fake(), fake(), fake(), None, None, fake(16),
                                     nat.workspace_size(c0), None) == nat.MOE_ERR_INVALID_ARG
    # misaligned codes
    assert fp8_raw(cfg(), w=nat.MoeFp8Experts(W1=4096 + 8, W1_scale=4096, Wu=4096, Wu_scale=4096, W2=4096,
                                              W2_scale=4096)) == nat.MOE_ERR_INVALID_ARG
    # the row quantizer
    L = nat.lib()
    assert L.moe_quantize_rows_e4m3(fake(), 4, 12, 12, fake(), 12, fake(), None) == nat.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize_rows_e4m3(fake(), 4, 16, 8, fake(), 16, fake(), None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_e4m3(fake(), 4, 16, 16, fake(), 12, fake(), None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_e4m3(None, 4, 16, 16, fake(), 16, fake(), None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_e4m3(None, 0, 16, 16, None, 16, None, None) == nat.MOE_OK


def test_mx_entry_points_check_arguments():
    L = nat.lib()
    # configuration: bf16, K dimensions multiples of 128, sld a multiple of 16 holding every K / 32
    assert nat.grouped_ffn_mx_workspace_size(cfg(), 16) > 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(dtype="f32"), 16) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(d_model=192), 16) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(d_ff=320), 16) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(d_ff_shared=64), 16) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(d_ff=768), 16) == 0       # 768 / 32 = 24 bytes > 16
    assert nat.grouped_ffn_mx_workspace_size(cfg(d_ff=768), 32) > 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(), 8) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(), 24) == 0
    assert nat.grouped_ffn_mx_workspace_size(cfg(E=300), 16) == 0
    assert nat.mx_sld(cfg(d_ff=768)) == 32 and nat.mx_sld(cfg()) == 16
    c = cfg()
    n = nat.grouped_ffn_mx_workspace_size(c, 16)

    def raw(w, **null):
        args = dict(x8p=fake(), xsp=fake(), off=fake(), rg=fake())
        rest = dict(b1=None, b2=None, x8=None, xs=None, y=fake())
        for k in null:
            (args if k in args else rest)[k] = None
        return L.moe_grouped_ffn_mx(ctypes.byref(c), *args.values(), ctypes.byref(w) if w is not None else None,
                                    *rest.values(), fake(16), n, None)

    full = dict(W1=4096, W1_scale=4096, Wu=4096, Wu_scale=4096, W2=4096, W2_scale=4096, sld=16)
    assert raw(None) == nat.MOE_ERR_INVALID_ARG
    assert raw(nat.MoeMxExperts(**dict(full, Wu_scale=None))) == nat.MOE_ERR_INVALID_ARG    # SwiGLU W_up scales
    assert "Wu_scale" in nat.last_error_detail()
    assert raw(nat.MoeMxExperts(**full), xsp=None) == nat.MOE_ERR_INVALID_ARG
    assert raw(nat.MoeMxExperts(**dict(full, W2_scale=4096 + 8))) == nat.MOE_ERR_INVALID_ARG  # misaligned
    assert raw(nat.MoeMxExperts(**dict(full, sld=8))) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_grouped_ffn_mx(ctypes.byref(c), fake(), fake(), fake(), fake(), ctypes.byref(nat.MoeMxExperts(**full)),
                                None, None, None, None, fake(), fake(16), n - 256, None) == nat.MOE_ERR_WORKSPACE
    # the MX row quantizer
    assert L.moe_quantize_rows_mx(fake(), 4, 48, 48, fake(), 48, fake(), 2, None) == nat.MOE_ERR_UNSUPPORTED
    assert L.moe_quantize_rows_mx(fake(), 4, 64, 64, fake(), 64, fake(), 1, None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_mx(fake(), 4, 64, 60, fake(), 64, fake(), 2, None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_mx(None, 4, 64, 64, fake(), 64, fake(), 2, None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_quantize_rows_mx(None, 0, 64, 64, None, 64, None, 2, None) == nat.MOE_OK


def test_router_freeze_checks_arguments():
    L = nat.lib()
    c = cfg()
    n = nat.workspace_size(c)
    assert L.moe_router_freeze(ctypes.byref(c), None, fake(16), n, None) == nat.MOE_ERR_INVALID_ARG
    assert L.moe_router_freeze(ctypes.byref(c), fake(), None, n, None) == nat.MOE_ERR_WORKSPACE
    assert L.moe_router_freeze(ctypes.byref(c), fake(), fake(16), n - 1, None) == nat.MOE_ERR_WORKSPACE
    c32 = cfg(dtype="f32")                                   # nothing to split for fp32 layers
    assert L.moe_router_freeze(ctypes.byref(c32), fake(), fake(16), nat.workspace_size(c32), None) == nat.MOE_OK


def test_workspace_view_addresses():
    # a host-only call: addresses inside the workspace, in increasing order,
    # aligned for their element type, every region inside ws_bytes
    for c in (cfg(T=300), cfg(T=300, d_ff_shared=64), cfg(T=64, dtype="f32"), cfg(T=0)):
        base, n = 1 << 20, nat.workspace_size(c)
        v = nat.MoeWsView()
        assert nat.lib().moe_workspace_view(ctypes.byref(c), ctypes.c_void_p(base), n, ctypes.byref(v)) == nat.MOE_OK
        T, d, E, k = c.T, c.d_model, c.E, c.top_k
        esz = 2 if c.dtype == nat.MOE_BF16 else 4
        rows = nat.perm_rows(c)
        regions = [(v.kept, 4 * E), (v.offsets, 4 * (E + 1)), (v.row_of, 4 * T * k), (v.row_token, 4 * T * k),
                   (v.row_gate, 4 * T * k), (v.x_perm, esz * T * k * d), (v.H, esz * rows * v.h_stride),
                   (v.y_perm, esz * rows * d)]
        assert v.h_stride == max(c.d_ff, c.d_ff_shared)
        end = base + 256                               # after the status header
        for addr, nbytes in regions:
            assert addr % 256 == 0 and addr >= end
            end = addr + nbytes
        assert end <= base + n
    c = cfg()
    v = nat.MoeWsView()
    L = nat.lib()
    assert L.moe_workspace_view(ctypes.byref(c), ctypes.c_void_p(4096), nat.workspace_size(c) - 1,
                                ctypes.byref(v)) == nat.MOE_ERR_WORKSPACE
    assert L.moe_workspace_view(ctypes.byref(c), ctypes.c_void_p(4096 + 8), nat.workspace_size(c),
                                ctypes.byref(v)) == nat.MOE_ERR_WORKSPACE
    assert L.moe_workspace_view(ctypes.byref(c), ctypes.c_void_p(4096), nat.workspace_size(c),
                                None) == nat.MOE_ERR_INVALID_ARG


def test_ep_grouped_ffn_host_checks():
    L = nat.lib()
    c = nat.make_config(0, 64, 4, 64, 1)
    assert L.moe_ep_workspace_size(ctypes.byref(c), 3, 100) == 256 + 100 * 64 * 2
    assert L.moe_ep_workspace_size(ctypes.byref(c), 64, 0) > 0                 # 256 groups
    assert L.moe_ep_workspace_size(ctypes.byref(c), 65, 0) == 0                 # 260 groups
    assert L.moe_ep_workspace_size(ctypes.byref(c), 0, 10) == 0
    assert L.moe_ep_workspace_size(ctypes.byref(nat.make_config(0, 60, 4, 64, 1)), 1, 10) == 0
    ws = fake(16)
    n = L.moe_ep_workspace_size(ctypes.byref(c), 2, 10)
    args = [fake(), 10, fake(), fake(), fake(), None, fake(), fake(), None, fake()]
    assert L.moe_ep_grouped_ffn(ctypes.byref(c), 2, *args, ws, n - 1, None) == nat.MOE_ERR_WORKSPACE
    assert L.moe_ep_grouped_ffn(ctypes.byref(c), 2, None, *args[1:], ws, n, None) == nat.MOE_ERR_INVALID_ARG
    bad = list(args)
    bad[6] = None                                       # SwiGLU without W_up
    assert L.moe_ep_grouped_ffn(ctypes.byref(c), 2, *bad, ws, n, None) == nat.MOE_ERR_INVALID_ARG
    # no rows: nothing to do, nothing launched
    assert L.moe_ep_grouped_ffn(ctypes.byref(c), 2, fake(), 0, None, None, None, None, None, None, None, None,
                                ws, 256, None) == nat.MOE_OK


def test_forward_train_checks_arguments():
    # the backward workspace is checked before anything runs
    L = nat.lib()
    c = cfg(d_model=128, d_ff=256)
    n = nat.workspace_size(c)
    nb = nat.backward_workspace_size(c)
    args = [fake(), fake(), None, None, fake(), None, fake(), fake(), None, None, None, None, fake(), fake(), fake(),
            fake(), fake(), fake(), fake(), None, None]
    call = lambda cc, bws, bn: L.moe_forward_train(ctypes.byref(cc), *args, fake(16), n, bws, bn, None)
    assert call(c, None, nb) == nat.MOE_ERR_WORKSPACE
    assert call(c, ctypes.c_void_p(4096 + 64), nb) == nat.MOE_ERR_WORKSPACE     # not 256-byte aligned
    assert call(c, fake(32), nb - 1) == nat.MOE_ERR_WORKSPACE
    c32 = cfg(dtype="f32")                                   # no backward pass for fp32 layers
    assert call(c32, fake(32), nb) == nat.MOE_ERR_UNSUPPORTED
    c96 = cfg(d_model=96)                                    # d_model not a multiple of 64
    assert call(c96, fake(32), nb) == nat.MOE_ERR_UNSUPPORTED
