"""The INT4 decode the GPU kernels use, modelled on the CPU.

A nibble u (= q + 8) placed in the low mantissa bits of bf16 128 (bits
0x4300) reads as 128 + u; subtracting 136 in bf16 is exact (the difference
is an integer in [-8, 7]) and one bf16 multiply by the group scale rounds
q * s once to nearest even -- so the decode gives bf16_rn(q * s), the
oracle's INT4 weight value, for every nibble and every bf16 scale whose
products stay normal.  Masking a code word shifted by 4j with 0x000F000F
yields inputs (j, j + 4) in one bf16x2 word; byte permutes pair the
neighbours (0,1) (2,3) (4,5) (6,7).  Checked here with exact arithmetic
(float64 for the products, torch's bf16 conversion for the rounding)
against the definition, nibble by nibble."""
import numpy as np
import torch

import oracle


def bf16_val(bits):
    return (np.asarray(bits, np.uint32) << 16).view(np.float32).astype(np.float64)


def bf16_rn(v):
    return torch.tensor(np.asarray(v, np.float64)).to(torch.float32).to(torch.bfloat16).view(torch.int16).numpy().astype(
        np.uint16)


def byte_perm(a, b, sel):
    src = [(a >> (8 * i)) & 255 for i in range(4)] + [(b >> (8 * i)) & 255 for i in range(4)]
    return sum(src[(sel >> (4 * i)) & 7] << (8 * i) for i in range(4))


def decode_word(word, s_bits):
    s = bf16_val(s_bits)
    t = []
    for j in range(4):
        x = ((word >> (4 * j)) & 0x000F000F) | 0x43004300
        halves = []
        for h in (x & 0xFFFF, x >> 16):
            q = bf16_val(h) - 136.0                      # exact: an integer in [-8, 7]
            assert q == int(q) and -8 <= q <= 7
            halves.append(int(bf16_rn(q * s)))           # one rounding of the exact product
        t.append(halves[0] | (halves[1] << 16))
    o = [byte_perm(t[0], t[1], 0x5410), byte_perm(t[2], t[3], 0x5410),
         byte_perm(t[0], t[1], 0x7632), byte_perm(t[2], t[3], 0x7632)]
    out = []
    for w in o:
        out += [w & 0xFFFF, w >> 16]
    return out


def test_magic_number_reads_128_plus_nibble():
    for u in range(16):
        assert bf16_val(0x4300 | u) == 128 + u
    assert bf16_val(0x4308) == 136.0


def test_decode_matches_the_definition():
    rng = np.random.default_rng(7)
    words = [0x76543210, 0xFEDCBA98, 0x0F0F0F0F, 0xF0F0F0F0] + [int(w) for w in rng.integers(0, 2 ** 32, 300)]
    scales = [0x3F80, 0x3C00, 0x4100, 0x3B2A, 0x3DCC] + [int(b) for b in rng.integers(0x2000, 0x5F00, 40)]
    for s_bits in scales:
        s = bf16_val(s_bits)
        for word in words:
            got = decode_word(word, s_bits)
            want = [int(bf16_rn((((word >> (4 * i)) & 15) - 8) * s)) for i in range(8)]
            assert got == want, (hex(word), hex(s_bits))


def test_decode_agrees_with_the_oracle_values():
    # the oracle's INT4 weight value of a packed byte pair, for a sample of scales
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 256, (4, 64)).astype(np.uint8)           # 4 rows of 128 inputs
    scale_bits = rng.integers(0x3A00, 0x4000, (4, 1)).astype(np.uint16)
    ref = oracle.w4_dequant(codes, scale_bits)
    for r in range(4):
        words = codes[r].view(np.uint32)
        got = []
        for w in words:
            got += decode_word(int(w), int(scale_bits[r, 0]))
        np.testing.assert_array_equal(bf16_val(np.array(got, np.uint32)), ref[r])
