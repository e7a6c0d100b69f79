"""The seeded input generator (CPU): the same seed gives the same tensors,
every tensor has its own stream, and the FP8 expert weights are finite e4m3
codes with per-channel scales in U(0.5, 1.5) / sqrt(fan_in)."""
import math

import numpy as np
import torch

from mixture_experts_layer_49_b200 import synthetic as syn

WL = syn.Workload("gen", T=48, d_model=64, E=6, d_ff=32, top_k=2, d_ff_shared=16, score="sigmoid",
                  sel_bias_std=0.1)


def test_generate_is_deterministic_and_streams_differ():
    a = syn.generate(WL, "cpu", seed=3)
    b = syn.generate(WL, "cpu", seed=3)
    c = syn.generate(WL, "cpu", seed=4)
    for key in ("x", "Wr", "W1", "Wu", "W2", "Wsg", "Wsu", "Wsd", "sel_bias"):
        assert torch.equal(a[key], b[key]), key
        assert not torch.equal(a[key], c[key]), key
    assert not torch.equal(a["W1"].float(), a["Wu"].float())
    assert not torch.equal(a["W1"][0].float(), a["W1"][1].float())


def test_fp8_experts_are_finite_codes_with_channel_scales():
    w = syn.generate_fp8_experts(WL, "cpu", seed=5)
    w2 = syn.generate_fp8_experts(WL, "cpu", seed=5)
    fan_in = {"W1": WL.d_model, "Wu": WL.d_model, "W2": WL.d_ff, "Wsg": WL.d_model, "Wsu": WL.d_model,
              "Wsd": WL.d_ff_shared}
    for key, fin in fan_in.items():
        codes, scale = w[key], w[key + "_scale"]
        assert codes.dtype == torch.uint8 and scale.dtype == torch.float32
        assert torch.equal(codes, w2[key]) and torch.equal(scale, w2[key + "_scale"])
        c = codes.numpy()
        assert not np.any((c & 0x7F) == 0x7F), key                        # no NaN codes
        assert scale.shape == codes.shape[:-1]
        s = scale.numpy() * math.sqrt(fin)
        assert s.min() >= 0.5 - 1e-6 and s.max() <= 1.5 + 1e-6, key
        # the dequantized weights have about unit variance times 1/fan_in
        v = codes.view(torch.float8_e4m3fn).float().numpy()
        assert 0.8 < float(np.std(v)) < 1.2, key
